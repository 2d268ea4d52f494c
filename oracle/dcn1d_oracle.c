/*
 * dcn1d_oracle.c -- plain, slow CPU oracle for the forward pass of 1D
 * deformable convolution (DeformConv1d, optional DCNv2 modulation mask).
 *
 * TEST INFRASTRUCTURE.  Only the tests, the smoke check and the bench's CPU
 * baseline may load this library.  It shares no code, header or constant with
 * the CUDA path and never reads anything the CUDA path produced.
 *
 * What it computes is the plain definition, written out with no blocking,
 * fusion or reordering:
 *
 *   out[b,co,l] = bias[co]
 *     + sum_{ci in conv group of co} sum_{k<K}
 *         W[co, ci - c0, k] * m[b,g(ci),l,k]
 *           * ((1-f) * X(b,ci,i0) + f * X(b,ci,i0+1))
 *
 * Sources (page title, section):
 *  - "conv1d" operator page (HNDL), "Description": the cross-correlation
 *    out = bias + sum_{ci,k} weight[co,ci,k] * x[b,ci,l*stride-padding+k*dilation];
 *    "Shape": the output-length closed form; "Axis convention": [B,C,L] and the
 *    meaning of groups; weight is [C_out, C_in/groups, K], bias is [C_out].
 *  - "A Detailed Explanation of the Calculation Workflow for Dilated
 *    Convolution and Deformable Convolution", "Deformable Convolution": each
 *    tap reads x at p0 + pn + delta_pn; "Step 2: Deformable Sampling": the
 *    interpolation weights are the fractional part and one minus it (the 1D
 *    case of the bilinear weights).
 *  - "dc1d (DeformConv1d)", "Usage / DeformConv1d": offsets are
 *    [B, offset_groups, L_out, K], offset_groups divides C_in, taps are
 *    constrained to their own receptive field unless unconstrained=True;
 *    "Modulation (DCNv2)": the mask has the offsets' shape, scales each
 *    sampled value and is applied as given.
 *  - "The document of torchvision.ops.deform_conv2d is not clear"
 *    (torchvision issue 3673), the kh=kw=1 demo: samples that fall outside
 *    the signal read zero; all channels of an offset group share offsets.
 *
 * Readings where the pages are silent (each one is listed in the design notes):
 *  - Receptive field of output l: [l*s - p, l*s - p + d*(K-1)]; in constrained
 *    mode the sampling position is clamped to it BEFORE the floor.
 *  - Offset group of channel ci: ci / (C_in / offset_groups) (contiguous blocks).
 *  - Padding "valid" is 0 and "same" (stride 1) is d(K-1)/2 zeros on the left and the
 *    rest on the right, as nn.Conv1d does (the dc1d page uses both strings and says its
 *    output length is nn.Conv1d's closed form); `padding` is the left side, and
 *    `padding_right` enters only the output length.
 *  - Sampling position: pos = (float)base + off in IEEE float32 with round to
 *    nearest; i0 = floor(pos); f = pos - (float)i0 in float32.  The
 *    interpolation and the sums are then done in double.
 *  - Build with -ffp-contract=off and without fast-math so that the float32
 *    steps round exactly as written.
 *
 * Inputs are float32 arrays (bf16 inputs are widened exactly by the caller).
 * Precondition: offsets are finite and |pos| < 2^24.
 */
#include <math.h>
#include <stddef.h>
#include <stdint.h>
#ifdef _OPENMP
#include <omp.h>
#endif

typedef struct {
    int64_t B, C_in, L_in, C_out, K, L_out;
    int64_t stride, padding, dilation, groups, offset_groups;
    int unconstrained;
    int64_t padding_right;   /* zeros after the signal; `padding` is the left side */
} oracle_shape;

/* "conv1d", "Shape" and "Description": L_out = floor((L_in + 2p - d(K-1) - 1)/s + 1),
 * here with the padding of each side separate: 2p -> pl + pr ("same" padding of the dc1d
 * page pads d(K-1)/2 on the left and the rest on the right, as nn.Conv1d does).
 * Returns -1 for out-of-range arguments or when the length would be < 1. */
static int64_t out_length_lr(int64_t L_in, int64_t K, int64_t s, int64_t pl, int64_t pr,
                             int64_t d)
{
    if (L_in < 1 || K < 1 || s < 1 || pl < 0 || pr < 0 || d < 1)
        return -1;
    int64_t num = L_in + pl + pr - d * (K - 1) - 1;
    if (num < 0)          /* then floor(num/s + 1) <= 0 */
        return -1;
    return num / s + 1;   /* num >= 0: integer division is the floor */
}

int64_t oracle_out_length(int64_t L_in, int64_t K, int64_t s, int64_t p, int64_t d)
{
    return out_length_lr(L_in, K, s, p, p, d);
}

int64_t oracle_out_length_lr(int64_t L_in, int64_t K, int64_t s, int64_t pl, int64_t pr,
                             int64_t d)
{
    return out_length_lr(L_in, K, s, pl, pr, d);
}

/* One tap's sampling position: the undeformed tap l*s - p + k*d plus the
 * learned offset (deformable-convolution formula, 1D), clamped in constrained
 * mode, split into its integer neighbour i0 and fraction f.  If gate is not
 * NULL it receives the clamp's derivative (backward): 0 when the clamp moved
 * the position, 1 otherwise (bounds included). */
static void sample_position(int64_t l, int64_t k, float off, const oracle_shape *S,
                            int64_t *i0, float *f, double *gate)
{
    int64_t start = l * S->stride - S->padding;
    int64_t base = start + k * S->dilation;
    float pos = (float)base + off;
    if (gate)
        *gate = 1.0;
    if (!S->unconstrained) {
        float lo = (float)start;
        float hi = (float)(start + S->dilation * (S->K - 1));
        if (gate && (pos < lo || pos > hi))
            *gate = 0.0;
        if (pos < lo) pos = lo;
        if (pos > hi) pos = hi;
    }
    float fl = floorf(pos);
    *i0 = (int64_t)fl;
    *f = pos - (float)(*i0);
}

/* x with zero fill outside [0, L_in - 1]. */
static double x_at(const float *x, const oracle_shape *S, int64_t b, int64_t ci, int64_t i)
{
    if (i < 0 || i >= S->L_in)
        return 0.0;
    return (double)x[(b * S->C_in + ci) * S->L_in + i];
}

/* One output element, by the definition above. */
static double output_point(const float *x, const float *off, const float *mask,
                           const float *w, const float *bias, const oracle_shape *S,
                           int64_t b, int64_t co, int64_t l)
{
    int64_t cin_g = S->C_in / S->groups;      /* input channels per conv group  */
    int64_t cout_g = S->C_out / S->groups;    /* output channels per conv group */
    int64_t cin_per_og = S->C_in / S->offset_groups;
    int64_t g = co / cout_g;
    double acc = bias ? (double)bias[co] : 0.0;
    for (int64_t c = 0; c < cin_g; ++c) {
        int64_t ci = g * cin_g + c;
        int64_t og = ci / cin_per_og;
        for (int64_t k = 0; k < S->K; ++k) {
            int64_t oidx = ((b * S->offset_groups + og) * S->L_out + l) * S->K + k;
            int64_t i0;
            float f;
            sample_position(l, k, off[oidx], S, &i0, &f, NULL);
            double v = (1.0 - (double)f) * x_at(x, S, b, ci, i0) + (double)f * x_at(x, S, b, ci, i0 + 1);
            if (mask)
                v *= (double)mask[oidx];
            acc += (double)w[(co * cin_g + c) * S->K + k] * v;
        }
    }
    return acc;
}

static int check_shape(const oracle_shape *S)
{
    if (S->B < 1 || S->C_in < 1 || S->C_out < 1 || S->K < 1 || S->L_in < 1)
        return 1;
    if (S->groups < 1 || S->C_in % S->groups || S->C_out % S->groups)
        return 1;
    if (S->offset_groups < 1 || S->C_in % S->offset_groups)
        return 1;
    if (out_length_lr(S->L_in, S->K, S->stride, S->padding, S->padding_right, S->dilation) !=
        S->L_out)
        return 1;
    return 0;
}

/* Every output: out[B, C_out, L_out] in double.  Returns 0, or 1 on bad shape. */
int oracle_forward(const float *x, const float *off, const float *mask, const float *w,
                   const float *bias, int64_t B, int64_t C_in, int64_t L_in, int64_t C_out,
                   int64_t K, int64_t L_out, int64_t stride, int64_t padding,
                   int64_t padding_right, int64_t dilation, int64_t groups,
                   int64_t offset_groups, int unconstrained, double *out)
{
    oracle_shape S = {B, C_in, L_in, C_out, K, L_out, stride, padding,
                      dilation, groups, offset_groups, unconstrained, padding_right};
    if (check_shape(&S))
        return 1;
#pragma omp parallel for collapse(2) schedule(dynamic, 1)
    for (int64_t b = 0; b < B; ++b)
        for (int64_t co = 0; co < C_out; ++co)
            for (int64_t l = 0; l < L_out; ++l)
                out[(b * C_out + co) * L_out + l] = output_point(x, off, mask, w, bias, &S, b, co, l);
    return 0;
}

/* Selected outputs only: points is [n, 3] of (b, co, l); out is [n]. */
int oracle_forward_points(const float *x, const float *off, const float *mask, const float *w,
                          const float *bias, int64_t B, int64_t C_in, int64_t L_in,
                          int64_t C_out, int64_t K, int64_t L_out, int64_t stride,
                          int64_t padding, int64_t padding_right, int64_t dilation,
                          int64_t groups, int64_t offset_groups, int unconstrained,
                          const int64_t *points, int64_t n, double *out)
{
    oracle_shape S = {B, C_in, L_in, C_out, K, L_out, stride, padding,
                      dilation, groups, offset_groups, unconstrained, padding_right};
    if (check_shape(&S))
        return 1;
    for (int64_t i = 0; i < n; ++i) {
        int64_t b = points[3 * i], co = points[3 * i + 1], l = points[3 * i + 2];
        if (b < 0 || b >= B || co < 0 || co >= C_out || l < 0 || l >= L_out)
            return 2;
    }
#pragma omp parallel for schedule(dynamic, 16)
    for (int64_t i = 0; i < n; ++i)
        out[i] = output_point(x, off, mask, w, bias, &S, points[3 * i], points[3 * i + 1],
                              points[3 * i + 2]);
    return 0;
}

/* The integer neighbour and fraction of every (b, g, l, k) tap. */
int oracle_sample_index(const float *off, int64_t B, int64_t G, int64_t L_in, int64_t K,
                        int64_t L_out, int64_t stride, int64_t padding, int64_t dilation,
                        int unconstrained, int32_t *i0_out, float *f_out)
{
    oracle_shape S = {B, G, L_in, G, K, L_out, stride, padding, dilation, 1, G, unconstrained,
                      padding};
    if (oracle_out_length(L_in, K, stride, padding, dilation) != L_out)
        return 1;
    int64_t n = B * G * L_out * K;
#pragma omp parallel for schedule(static)
    for (int64_t t = 0; t < n; ++t) {
        int64_t k = t % K;
        int64_t l = (t / K) % L_out;
        int64_t i0;
        float f;
        sample_position(l, k, off[t], &S, &i0, &f, NULL);
        i0_out[t] = (int32_t)i0;
        f_out[t] = f;
    }
    return 0;
}

/* Threads an OpenMP region of this library will use. */
int oracle_threads(void)
{
#ifdef _OPENMP
    return omp_get_max_threads();
#else
    return 1;
#endif
}

void oracle_set_threads(int n)
{
#ifdef _OPENMP
    if (n > 0)
        omp_set_num_threads(n);
#else
    (void)n;
#endif
}

/* ------------------------------------------------------------------ backward
 *
 * Gradients of the forward above with respect to every input, for an upstream
 * gradient gout[B, C_out, L_out] (the loss is sum(gout * out)).
 *
 * Source: "dc1d (DeformConv1d)" page, opening paragraph: the layer is plain
 * tensor code and is trained through torch.autograd, so its gradient is the
 * derivative of the forward as written; the "Demo notebook" note checks the
 * offset gradient against a finite difference.  Writing v = (1-f) X(i0) + f X(i0+1)
 * and dv(b,ci,l,k) = sum_{co in the conv group of ci} gout[b,co,l] W[co,ci-c0,k]:
 *
 *   grad_bias[co]        = sum_{b,l} gout[b,co,l]
 *   grad_weight[co,c,k]  = sum_{b,l} gout[b,co,l] * m * v
 *   grad_x[b,ci,i0]     += m (1-f) dv,   grad_x[b,ci,i0+1] += m f dv   (inside [0, L_in) only)
 *   grad_mask[b,g,l,k]   = sum_{ci in offset group g} v dv
 *   grad_offsets[b,g,l,k]= sum_{ci in offset group g} m (X(i0+1) - X(i0)) dv * gate
 *
 * Readings (listed in the design notes): floor() contributes nothing (the
 * slope inside a unit cell is X(i0+1) - X(i0), the right-hand one at an
 * integer position); in constrained mode the clamp passes the offset gradient
 * when lo <= pos <= hi (bounds included, as torch.clamp does) and stops it
 * outside (gate = 0 there); the position's float32 rounding counts as exact.
 * Every output array may be NULL (skipped); all are float64.
 */
int oracle_backward(const float *x, const float *off, const float *mask, const float *w,
                    const float *gout, int64_t B, int64_t C_in, int64_t L_in, int64_t C_out,
                    int64_t K, int64_t L_out, int64_t stride, int64_t padding,
                    int64_t padding_right, int64_t dilation, int64_t groups,
                    int64_t offset_groups, int unconstrained, double *gx, double *goff,
                    double *gmask, double *gw, double *gbias)
{
    oracle_shape S = {B, C_in, L_in, C_out, K, L_out, stride, padding,
                      dilation, groups, offset_groups, unconstrained, padding_right};
    if (check_shape(&S))
        return 1;
    const int64_t cin_g = C_in / groups, cout_g = C_out / groups;
    const int64_t cin_per_og = C_in / offset_groups;

    /* grad_x, grad_offsets, grad_mask: one (b, offset group) per iteration owns
     * the x rows of its channels and its offset/mask entries. */
#pragma omp parallel for collapse(2) schedule(dynamic, 1)
    for (int64_t b = 0; b < B; ++b)
        for (int64_t og = 0; og < offset_groups; ++og) {
            for (int64_t ci = og * cin_per_og; ci < (og + 1) * cin_per_og; ++ci)
                if (gx)
                    for (int64_t i = 0; i < L_in; ++i)
                        gx[(b * C_in + ci) * L_in + i] = 0.0;
            for (int64_t l = 0; l < L_out; ++l)
                for (int64_t k = 0; k < K; ++k) {
                    int64_t oidx = ((b * offset_groups + og) * L_out + l) * K + k;
                    int64_t i0;
                    float f;
                    double gate;
                    sample_position(l, k, off[oidx], &S, &i0, &f, &gate);
                    double m = mask ? (double)mask[oidx] : 1.0;
                    double sum_off = 0.0, sum_mask = 0.0;
                    for (int64_t ci = og * cin_per_og; ci < (og + 1) * cin_per_og; ++ci) {
                        int64_t g = ci / cin_g, c = ci - g * cin_g;
                        double dv = 0.0;
                        for (int64_t co = g * cout_g; co < (g + 1) * cout_g; ++co)
                            dv += (double)gout[(b * C_out + co) * L_out + l] *
                                  (double)w[(co * cin_g + c) * K + k];
                        double x0 = x_at(x, &S, b, ci, i0), x1 = x_at(x, &S, b, ci, i0 + 1);
                        if (gx) {
                            if (i0 >= 0 && i0 < L_in)
                                gx[(b * C_in + ci) * L_in + i0] += m * (1.0 - (double)f) * dv;
                            if (i0 + 1 >= 0 && i0 + 1 < L_in)
                                gx[(b * C_in + ci) * L_in + i0 + 1] += m * (double)f * dv;
                        }
                        sum_off += m * (x1 - x0) * dv;
                        sum_mask += ((1.0 - (double)f) * x0 + (double)f * x1) * dv;
                    }
                    if (goff)
                        goff[oidx] = sum_off * gate;
                    if (gmask)
                        gmask[oidx] = sum_mask;
                }
        }

    /* grad_weight: one (co, c) per iteration. */
    if (gw) {
#pragma omp parallel for collapse(2) schedule(dynamic, 1)
        for (int64_t co = 0; co < C_out; ++co)
            for (int64_t c = 0; c < cin_g; ++c) {
                int64_t g = co / cout_g, ci = g * cin_g + c, og = ci / cin_per_og;
                for (int64_t k = 0; k < K; ++k) {
                    double acc = 0.0;
                    for (int64_t b = 0; b < B; ++b)
                        for (int64_t l = 0; l < L_out; ++l) {
                            int64_t oidx = ((b * offset_groups + og) * L_out + l) * K + k;
                            int64_t i0;
                            float f;
                            sample_position(l, k, off[oidx], &S, &i0, &f, NULL);
                            double v = (1.0 - (double)f) * x_at(x, &S, b, ci, i0) +
                                       (double)f * x_at(x, &S, b, ci, i0 + 1);
                            if (mask)
                                v = v * (double)mask[oidx];
                            acc += (double)gout[(b * C_out + co) * L_out + l] * v;
                        }
                    gw[(co * cin_g + c) * K + k] = acc;
                }
            }
    }

    if (gbias)
        for (int64_t co = 0; co < C_out; ++co) {
            double acc = 0.0;
            for (int64_t b = 0; b < B; ++b)
                for (int64_t l = 0; l < L_out; ++l)
                    acc += (double)gout[(b * C_out + co) * L_out + l];
            gbias[co] = acc;
        }
    return 0;
}

/* ------------------------------------------------------------------ packed trunk
 *
 * The offset (and mask) predictor of PackedDeformConv1d.  Sources: "dc1d
 * (DeformConv1d)" page, "PackedDeformConv1d": the layer computes its offsets
 * itself with a depthwise-separable convolution block; "Modulation (DCNv2)":
 * with modulated=True a second pointwise branch off the same depthwise trunk
 * predicts the mask and ends in a sigmoid.  The deformable-convolution article,
 * "Step 1: Offset Generation", makes the offset stage an ordinary convolution
 * over the input whose output channels are the offsets of every tap.
 *
 *   t[b,c,l]      = dw_b[c] + sum_k dw_w[c,k] * X(b, c, l*s - pl + k*d)
 *   off[b,g,l,k]  = off_b[g*K+k]  + sum_c off_w[g*K+k, c]  * t[b,c,l]
 *   mask[b,g,l,k] = sigmoid(mask_b[g*K+k] + sum_c mask_w[g*K+k, c] * t[b,c,l])
 *
 * Readings where the pages are silent (listed in the design notes): the
 * depthwise convolution takes the layer's own kernel size, stride, padding and
 * dilation (so it yields one offset vector per output position); nothing sits
 * between the depthwise and the pointwise convolution; pointwise output channel
 * g*K + k is the offset (mask) of tap k of offset group g.  Every bias may be NULL
 * (none); mask_w NULL means no mask branch.  Outputs are float64
 * [B, offset_groups, L_out, K].
 */
int oracle_packed_trunk(const float *x, const float *dw_w, const float *dw_b,
                        const float *off_w, const float *off_b, const float *mask_w,
                        const float *mask_b, int64_t B, int64_t C_in, int64_t L_in, int64_t K,
                        int64_t L_out, int64_t stride, int64_t padding, int64_t padding_right,
                        int64_t dilation, int64_t offset_groups, double *off_out,
                        double *mask_out)
{
    if (B < 0 || C_in < 1 || L_in < 0 || K < 1 || stride < 1 || dilation < 1 || padding < 0 ||
        padding_right < 0 || offset_groups < 1 || C_in % offset_groups != 0)
        return 1;
    if (L_out != out_length_lr(L_in, K, stride, padding, padding_right, dilation))
        return 1;
    const int64_t J = offset_groups * K;
#pragma omp parallel for collapse(2) schedule(static)
    for (int64_t b = 0; b < B; ++b)
        for (int64_t l = 0; l < L_out; ++l) {
            double t[C_in];
            /* the depthwise stage at output position l */
            for (int64_t c = 0; c < C_in; ++c) {
                double acc = dw_b ? (double)dw_b[c] : 0.0;
                for (int64_t k = 0; k < K; ++k) {
                    int64_t i = l * stride - padding + k * dilation;
                    double xv = (i >= 0 && i < L_in) ? (double)x[(b * C_in + c) * L_in + i] : 0.0;
                    acc += (double)dw_w[c * K + k] * xv;
                }
                t[c] = acc;
            }
            /* the pointwise projections */
            for (int64_t j = 0; j < J; ++j) {
                int64_t g = j / K, k = j % K;
                int64_t oidx = ((b * offset_groups + g) * L_out + l) * K + k;
                double z = off_b ? (double)off_b[j] : 0.0;
                for (int64_t c = 0; c < C_in; ++c)
                    z += (double)off_w[j * C_in + c] * t[c];
                off_out[oidx] = z;
                if (mask_w && mask_out) {
                    double zm = mask_b ? (double)mask_b[j] : 0.0;
                    for (int64_t c = 0; c < C_in; ++c)
                        zm += (double)mask_w[j * C_in + c] * t[c];
                    mask_out[oidx] = 1.0 / (1.0 + exp(-zm));
                }
            }
        }
    return 0;
}
