// The sampling step of the 1D deformable convolution: one tap's position.
//
// The undeformed tap of output l reads x at l*stride - padding + k*dilation
// ("conv1d" page, "Description"); deformable convolution adds the learned
// offset to it (the article "... Dilated Convolution and Deformable
// Convolution", section "Deformable Convolution": y(p0) = sum w(pn) x(p0+pn+dpn)).
// Unless unconstrained, the position is clamped to the tap's receptive field
// [l*stride - padding, l*stride - padding + dilation*(K-1)] (dc1d page,
// "Usage": each tap is constrained to its own receptive field).  The result is
// split into the integer neighbour i0 = floor(pos) and the fraction f, which
// weight the neighbours i0 and i0+1 by (1-f) and f (the 1D case of the
// bilinear weights in "Step 2: Deformable Sampling").
//
// Float32 with explicit round-to-nearest intrinsics, so that no contraction or
// reassociation changes the integer decision: every kernel and the
// dcn1d_sample_index entry point call this one function.
#pragma once

#include "common.cuh"

namespace dcn1d {

struct Tap {
    int i0;    // floor of the sampling position
    float f;   // position - i0, in [0, 1) for finite positions
};

// `start` = l*stride - padding, `span` = dilation*(K-1).
__device__ __forceinline__ Tap sample_tap(int start, int k, int dilation, int span, float off,
                                          bool unconstrained) {
    float pos = __fadd_rn(__int2float_rn(start + k * dilation), off);
    if (!unconstrained) {
        pos = fmaxf(pos, __int2float_rn(start));
        pos = fminf(pos, __int2float_rn(start + span));
    }
    Tap t;
    t.i0 = __float2int_rd(pos);
    t.f = __fsub_rn(pos, __int2float_rn(t.i0));
    return t;
}

// (1-f)*x[i0] + f*x[i0+1] with x zero outside [0, L).  Every access is bounds
// checked without overflow, whatever i0 is (NaN and huge offsets included).
template <class T>
__device__ __forceinline__ float lerp_row(const T *row, int L, Tap t) {
    float x0 = (t.i0 >= 0 && t.i0 < L) ? ld_f32(row + t.i0) : 0.0f;
    float x1 = (t.i0 >= -1 && t.i0 < L - 1) ? ld_f32(row + t.i0 + 1) : 0.0f;
    return __fadd_rn(__fmul_rn(__fsub_rn(1.0f, t.f), x0), __fmul_rn(t.f, x1));
}

}  // namespace dcn1d
