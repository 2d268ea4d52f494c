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
// Float32 with explicit rounding intrinsics, so that no contraction or
// reassociation changes the integer decision.  Two floors compute the same
// (i0, f) wherever both apply:
//  * tap_floor_exact: float->int conversion, valid for every |pos| < 2^31;
//  * tap_floor_fast: one round-down add of 1.5*2^23 (no conversion
//    instructions), exact for |pos| < 2^22.  For any other float (huge, inf,
//    NaN) it returns an i0 outside [-2^22, 2^22), i.e. outside every signal the
//    fast kernels accept (L_in <= 2^22), so both neighbours read zero.
#pragma once

#include "common.cuh"

namespace dcn1d {

struct Tap {
    int i0;    // floor of the sampling position
    float f;   // position - i0, in [0, 1) for finite positions
};

constexpr float kFloorMagic = 12582912.0f;        // 1.5 * 2^23
constexpr unsigned kFloorMagicBits = 0x4B400000u;  // its bit pattern
constexpr int kFastPosLimit = 1 << 22;            // |pos| below this: fast floor exact

__device__ __forceinline__ Tap tap_floor_exact(float pos) {
    Tap t;
    t.i0 = __float2int_rd(pos);
    t.f = __fsub_rn(pos, __int2float_rn(t.i0));
    return t;
}

// pos + M rounded down is M + floor(pos) when it stays in [2^23, 2^24), where
// floats are the integers; its bits minus M's bits are then floor(pos).
__device__ __forceinline__ Tap tap_floor_fast(float pos) {
    const float t = __fadd_rd(pos, kFloorMagic);
    Tap r;
    r.i0 = (int)(__float_as_uint(t) - kFloorMagicBits);
    r.f = __fsub_rn(pos, __fsub_rn(t, kFloorMagic));
    return r;
}

// Position of tap k of the output whose receptive field starts at `start`
// (= l*stride - padding); `span` = dilation*(K-1).
__device__ __forceinline__ float tap_position(int start, int k, int dilation, int span, float off,
                                             bool unconstrained) {
    float pos = __fadd_rn(__int2float_rn(start + k * dilation), off);
    if (!unconstrained) {
        pos = fmaxf(pos, __int2float_rn(start));
        pos = fminf(pos, __int2float_rn(start + span));
    }
    return pos;
}

__device__ __forceinline__ Tap sample_tap(int start, int k, int dilation, int span, float off,
                                          bool unconstrained) {
    return tap_floor_exact(tap_position(start, k, dilation, span, off, unconstrained));
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
