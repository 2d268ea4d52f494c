// Backward pass of the 1D deformable convolution: gradients of sum(grad_out * y)
// with respect to x, the offsets, the mask, the weight and the bias.
//
// The layer is trained through autograd on the forward as written ("dc1d
// (DeformConv1d)" page, opening paragraph; its demo notebook checks the offset
// gradient against a finite difference), so the backward is that derivative.
// With v = (1-f) x[i0] + f x[i0+1] the sampled value of tap (l, k) in channel
// ci and dv = sum_co W[co, ci, k] grad_out[b, co, l] over the conv group:
//   grad_weight[co, c, k] = sum_{b,l} grad_out[b, co, l] * m * v
//   grad_x[b, ci, i0]    += m (1-f) dv,    grad_x[b, ci, i0+1] += m f dv
//   grad_mask[b, g, l, k] = sum_{ci in offset group g} v dv
//   grad_offsets         = sum_{ci in g} m (x[i0+1] - x[i0]) dv   (0 where the
//                          constrained clamp moved the position)
//   grad_bias[co]         = sum_{b,l} grad_out[b, co, l]
//
// Kernels, fp32 arithmetic whatever the input type (16-bit problems contract 16-bit
// operands on the tensor cores with fp32 accumulation):
//  1. dcols[b, (c,k), l] = sum_co W[co, (c,k)] grad_out[b, co, l]: a batched GEMM
//     per (batch, conv group); 16-bit problems: the tensor-core GEMM of gemm_tc.cu on
//     K-major copies (grad_out transposed to [b][l][co], W per group to [(c,k)][co]),
//     otherwise on CUDA cores (64x64 tiles, 4x4 per thread);
//  2. the sampling gradient: one thread per (batch, 16-channel chunk, offset
//     group, tap, position) recomputes the tap's position once, then for its
//     channels scatters grad_x, sums the offset and mask gradients (atomics
//     into fp32 scratch: the order of those sums is not fixed) and writes the
//     sampled columns m*v that the weight gradient needs;
//  3. grad_weight = sum_b grad_out[b] cols[b]^T: the same GEMM kernel, summing
//     over the batch inside the tile loop (16-bit problems: the tensor-core GEMM on
//     16-bit columns); when that grid is small the batch sum is split across CTAs
//     into fp32 slices added in split order (a fixed order);
//  4. grad_bias: one block per channel, a fixed-order tree reduction;
//  5. the fp32 scratch of grad_x / grad_offsets / grad_mask is written out in
//     the input type.
#include <string.h>

#include "common.cuh"
#include "sampler.cuh"
#include "sm100.cuh"

namespace dcn1d {

namespace {

constexpr int kBM = 64, kBN = 64, kBKd = 16;   // GEMM tile
constexpr int kChunk = 16;                     // channels per sampling-gradient thread

// C[zb, zg][m][n] = sum_{r < R} sum_{kk < Kd} A[zb, zg, r][m][kk] * B[zb, zg, r][kk][n]
// with blockIdx.z = zb * ng + zg; every stride in elements.
struct GemmArgs {
    int M, N, Kd, R, ng;
    int64_t a_sm, a_sk, a_sb, a_sg, a_sr;
    int64_t b_sk, b_sn, b_sb, b_sg, b_sr;
    int64_t c_sm, c_sn, c_sb, c_sg;
};

// 64x64 output tile per 256 threads, 4x4 per thread; A_MC: A is contiguous along m
// (else along kk), B_NC: B is contiguous along n (else along kk) -- the tile loads
// run along the contiguous direction.
template <class TA, class TB, class TC, bool A_MC, bool B_NC>
__global__ void __launch_bounds__(256) gemm_kernel(const TA *__restrict__ A,
                                                   const TB *__restrict__ B, TC *__restrict__ C,
                                                   const GemmArgs g) {
    __shared__ __align__(16) float As[kBKd][kBM + 4];
    __shared__ __align__(16) float Bs[kBKd][kBN + 4];
    const int tid = threadIdx.x;
    const int m0 = blockIdx.y * kBM, n0 = blockIdx.x * kBN;
    const int zb = blockIdx.z / g.ng, zg = blockIdx.z - zb * g.ng;
    const TA *Az = A + zb * g.a_sb + zg * g.a_sg;
    const TB *Bz = B + zb * g.b_sb + zg * g.b_sg;
    const int tm = (tid / 16) * 4, tn = (tid % 16) * 4;
    float acc[4][4];
#pragma unroll
    for (int i = 0; i < 4; ++i)
#pragma unroll
        for (int j = 0; j < 4; ++j)
            acc[i][j] = 0.0f;
    for (int r = 0; r < g.R; ++r) {
        const TA *Ar = Az + r * g.a_sr;
        const TB *Br = Bz + r * g.b_sr;
        for (int k0 = 0; k0 < g.Kd; k0 += kBKd) {
#pragma unroll
            for (int i = 0; i < 4; ++i) {
                const int e = tid + i * 256;
                const int m = A_MC ? e % kBM : e / kBKd;
                const int kk = A_MC ? e / kBM : e % kBKd;
                const bool in = m0 + m < g.M && k0 + kk < g.Kd;
                As[kk][m] = in ? to_f32(Ar[(int64_t)(m0 + m) * g.a_sm + (int64_t)(k0 + kk) * g.a_sk])
                               : 0.0f;
                const int n = B_NC ? e % kBN : e / kBKd;
                const int kb = B_NC ? e / kBN : e % kBKd;
                const bool inb = n0 + n < g.N && k0 + kb < g.Kd;
                Bs[kb][n] = inb ? to_f32(Br[(int64_t)(k0 + kb) * g.b_sk + (int64_t)(n0 + n) * g.b_sn])
                                : 0.0f;
            }
            __syncthreads();
#pragma unroll
            for (int kk = 0; kk < kBKd; ++kk) {
                const float4 a = *reinterpret_cast<const float4 *>(&As[kk][tm]);
                const float4 b = *reinterpret_cast<const float4 *>(&Bs[kk][tn]);
                const float av[4] = {a.x, a.y, a.z, a.w}, bv[4] = {b.x, b.y, b.z, b.w};
#pragma unroll
                for (int i = 0; i < 4; ++i)
#pragma unroll
                    for (int j = 0; j < 4; ++j)
                        acc[i][j] = __fmaf_rn(av[i], bv[j], acc[i][j]);
            }
            __syncthreads();
        }
    }
    TC *Cz = C + zb * g.c_sb + zg * g.c_sg;
#pragma unroll
    for (int i = 0; i < 4; ++i)
#pragma unroll
        for (int j = 0; j < 4; ++j)
            if (m0 + tm + i < g.M && n0 + tn + j < g.N)
                Cz[(int64_t)(m0 + tm + i) * g.c_sm + (int64_t)(n0 + tn + j) * g.c_sn] =
                    from_f32<TC>(acc[i][j]);
}

template <class TA, class TB, class TC, bool A_MC, bool B_NC>
cudaError_t run_gemm(const TA *A, const TB *B, TC *C, const GemmArgs &g, int nz,
                     cudaStream_t stream) {
    const dim3 grid((g.N + kBN - 1) / kBN, (g.M + kBM - 1) / kBM, nz);
    gemm_kernel<TA, TB, TC, A_MC, B_NC><<<grid, 256, 0, stream>>>(A, B, C, g);
    return cudaGetLastError();
}

// out[i] = sum over s < S of part[s][i] in split order, written in the output type.
template <class T>
__global__ void __launch_bounds__(256) sum_splits_kernel(const float *part, T *out, int S,
                                                         int64_t n) {
    for (int64_t i = (int64_t)blockIdx.x * blockDim.x + threadIdx.x; i < n;
         i += (int64_t)gridDim.x * blockDim.x) {
        float acc = 0.0f;
        for (int s = 0; s < S; ++s)
            acc = __fadd_rn(acc, part[(int64_t)s * n + i]);
        out[i] = from_f32<T>(acc);
    }
}

struct SampArgs {
    Problem P;
    int cols_ld;                 // row stride of `cols` (L_out, or L_out padded to 4)
    int nchunk;                  // channel chunks per offset group
    int nlb;                     // blocks of kSgRows positions per (b, chunk, offset group)
    int win;                     // shared-memory grad_x window per channel (0: none)
    int margin;                  // window positions before the first receptive field
    const float *dcols;          // [B][C_in*K][L_out] or NULL
    float *cols;                 // [B][C_in*K][L_out] or NULL
    void *cols16;                // the same columns in the input's 16-bit type, or NULL
    float *gx, *goff, *gmask;    // fp32 scratch, each may be NULL
};

constexpr int kSgRows = 256;     // output positions per sampling-gradient block

// Block = (kSgRows consecutive positions l, channel chunk, offset group, b); thread = one
// position, looping over the taps k and the chunk's channels.  The grad_x scatter of all
// taps of the block's positions goes to a shared-memory window over the chunk's rows
// ([nc][win] fp32, positions w0 .. w0+win-1); taps outside it (unconstrained offsets past
// the margin) add to global memory directly, and the window is added to global memory
// once, element by element, at the end.  Six blocks an SM (40 registers): the loads in
// flight, not the instruction count, set this kernel's pace.
template <class T, bool MASK>
__global__ void __launch_bounds__(kSgRows, 6) sample_grad_kernel(const SampArgs a) {
    extern __shared__ float gxs[];
    const Problem &P = a.P;
    int64_t r = blockIdx.x;
    const int lb = (int)(r % a.nlb);
    r /= a.nlb;
    const int chunk = (int)(r % a.nchunk);
    r /= a.nchunk;
    const int og = (int)(r % P.offset_groups);
    const int b = (int)(r / P.offset_groups);
    const int l0 = lb * kSgRows;
    const int l = l0 + (int)threadIdx.x;
    const int c_begin = og * P.cin_per_og + chunk * kChunk;
    const int c_end = min(c_begin + kChunk, (og + 1) * P.cin_per_og);
    const int nc = c_end - c_begin;
    const bool window = a.gx && a.dcols && a.win > 0;
    const int W = a.win;
    const int w0 = l0 * P.stride - P.padding - a.margin;
    if (window) {
        for (int i = threadIdx.x; i < nc * W; i += blockDim.x)
            gxs[i] = 0.0f;
        __syncthreads();
    }
    if (l < P.L_out) {
        const int start = l * P.stride - P.padding;
        const int span = P.dilation * (P.K - 1);
        for (int k = 0; k < P.K; ++k) {
            const int64_t oidx = (((int64_t)b * P.offset_groups + og) * P.L_out + l) * P.K + k;
            const float off = ld_f32(static_cast<const T *>(P.off) + oidx);
            const float m = MASK ? ld_f32(static_cast<const T *>(P.mask) + oidx) : 1.0f;
            const float raw = __fadd_rn(__int2float_rn(start + k * P.dilation), off);
            // The clamp passes the gradient inside its closed range (NaN: no gradient).
            const bool gate = P.unconstrained ||
                              (raw >= __int2float_rn(start) && raw <= __int2float_rn(start + span));
            const Tap tp = sample_tap(start, k, P.dilation, span, off, P.unconstrained);
            const float mf = __fmul_rn(m, tp.f), m1f = __fmul_rn(m, __fsub_rn(1.0f, tp.f));
            const bool in0 = tp.i0 >= 0 && tp.i0 < P.L_in;
            const bool in1 = tp.i0 >= -1 && tp.i0 < P.L_in - 1;
            // window-relative neighbours (unsigned compares also reject NaN-free far taps)
            const int r0 = tp.i0 - w0;
            const bool win0 = window && r0 >= 0 && r0 < W;
            const bool win1 = window && r0 + 1 >= 0 && r0 + 1 < W;
            float s_off = 0.0f, s_mask = 0.0f;
            // The next channel's neighbours and column gradient are loaded while this
            // channel's are used, so two channels' global loads are in flight a thread.
            const T *row = static_cast<const T *>(P.x) + ((int64_t)b * P.C_in + c_begin) * P.L_in;
            const int64_t cstride = (int64_t)P.K * P.L_out;   // column rows between channels
            int64_t cidx = (((int64_t)b * P.C_in + c_begin) * P.K + k) * P.L_out + l;
            float nx0 = in0 ? ld_f32(row + tp.i0) : 0.0f;
            float nx1 = in1 ? ld_f32(row + tp.i0 + 1) : 0.0f;
            float ndv = a.dcols ? a.dcols[cidx] : 0.0f;
            for (int ci = c_begin; ci < c_end; ++ci, row += P.L_in, cidx += cstride) {
                const float x0 = nx0, x1 = nx1, dv = ndv;
                if (ci + 1 < c_end) {
                    nx0 = in0 ? ld_f32(row + P.L_in + tp.i0) : 0.0f;
                    nx1 = in1 ? ld_f32(row + P.L_in + tp.i0 + 1) : 0.0f;
                    ndv = a.dcols ? a.dcols[cidx + cstride] : 0.0f;
                }
                const float v = __fadd_rn(__fmul_rn(__fsub_rn(1.0f, tp.f), x0), __fmul_rn(tp.f, x1));
                if (a.cols)   // row (b, ci, k) of the columns, cols_ld elements apart
                    a.cols[(((int64_t)b * P.C_in + ci) * P.K + k) * a.cols_ld + l] =
                        __fmul_rn(m, v);
                if (sizeof(T) == 2 && a.cols16)
                    static_cast<T *>(a.cols16)[cidx] = from_f32<T>(__fmul_rn(m, v));
                if (a.dcols) {
                    if (a.gx) {
                        float *gxr = a.gx + ((int64_t)b * P.C_in + ci) * P.L_in;
                        float *wr = gxs + (ci - c_begin) * W;
                        if (in0) {
                            if (win0)
                                atomicAdd(wr + r0, __fmul_rn(m1f, dv));
                            else
                                atomicAdd(gxr + tp.i0, __fmul_rn(m1f, dv));
                        }
                        if (in1) {
                            if (win1)
                                atomicAdd(wr + r0 + 1, __fmul_rn(mf, dv));
                            else
                                atomicAdd(gxr + tp.i0 + 1, __fmul_rn(mf, dv));
                        }
                    }
                    s_off = __fmaf_rn(__fmul_rn(m, __fsub_rn(x1, x0)), dv, s_off);
                    s_mask = __fmaf_rn(v, dv, s_mask);
                }
            }
            if (a.dcols && a.goff && gate)
                atomicAdd(a.goff + oidx, s_off);
            if (a.dcols && a.gmask)
                atomicAdd(a.gmask + oidx, s_mask);
        }
    }
    if (window) {
        __syncthreads();
        // untouched (zero) entries add nothing: skipped
        for (int i = threadIdx.x; i < nc * W; i += blockDim.x) {
            const int c = i / W, w = i - c * W;
            const int pos = w0 + w;
            const float v = gxs[i];
            if (v != 0.0f && pos >= 0 && pos < P.L_in)
                atomicAdd(a.gx + ((int64_t)b * P.C_in + c_begin + c) * P.L_in + pos, v);
        }
    }
}

// dst[z][c][r] = src[z][r][c] for z < nz, r < R, c < Cc (16-bit elements): 32 x 32 tiles
// through shared memory, both sides coalesced.  Source rows are ld_src elements apart,
// destination rows ld_dst; z strides in elements.
template <class T>
__global__ void __launch_bounds__(256) transpose_kernel(const T *src, T *dst, int R, int Cc,
                                                        int64_t ld_src, int64_t ld_dst,
                                                        int64_t sz_src, int64_t sz_dst) {
    __shared__ T tile[32][33];
    const int z = blockIdx.z;
    const int r0 = blockIdx.y * 32, c0 = blockIdx.x * 32;
    const int tx = threadIdx.x % 32, ty = threadIdx.x / 32;   // 32 x 8
    const T *s = src + (int64_t)z * sz_src;
    T *d = dst + (int64_t)z * sz_dst;
    for (int i = ty; i < 32; i += 8)
        if (r0 + i < R && c0 + tx < Cc)
            tile[i][tx] = s[(int64_t)(r0 + i) * ld_src + c0 + tx];
    __syncthreads();
    for (int i = ty; i < 32; i += 8)
        if (c0 + i < Cc && r0 + tx < R)
            d[(int64_t)(c0 + i) * ld_dst + r0 + tx] = tile[tx][i];
}

// grad_bias[co] = sum over (b, l) of grad_out[b, co, l]: one block per channel,
// a fixed-order reduction.
template <class T>
__global__ void __launch_bounds__(256) bias_grad_kernel(const T *gout, T *gbias, int B,
                                                        int C_out, int L_out) {
    __shared__ float part[256];
    const int co = blockIdx.x;
    float s = 0.0f;
    // 16-byte loads where every row allows them (VE elements each), four in flight per
    // thread; each thread adds its elements in a fixed order
    constexpr int VE = 16 / (int)sizeof(T);
    if (L_out % VE == 0 && (reinterpret_cast<uintptr_t>(gout) & 15) == 0) {
        const int nv = L_out / VE;
        const int64_t n = (int64_t)B * nv;
        auto at = [&](int64_t i) {
            const int b = (int)(i / nv), j = (int)(i - (int64_t)b * nv);
            return reinterpret_cast<const uint4 *>(gout + ((int64_t)b * C_out + co) * L_out) + j;
        };
        auto add = [&](uint4 u) {
            const T *e = reinterpret_cast<const T *>(&u);
#pragma unroll
            for (int q = 0; q < VE; ++q)
                s = __fadd_rn(s, to_f32(e[q]));
        };
        int64_t i = threadIdx.x;
        for (; i + 3 * (int64_t)blockDim.x < n; i += 4 * (int64_t)blockDim.x) {
            const uint4 u0 = __ldg(at(i)), u1 = __ldg(at(i + blockDim.x)),
                        u2 = __ldg(at(i + 2 * blockDim.x)), u3 = __ldg(at(i + 3 * blockDim.x));
            add(u0);
            add(u1);
            add(u2);
            add(u3);
        }
        for (; i < n; i += blockDim.x)
            add(__ldg(at(i)));
    } else {
        for (int64_t i = threadIdx.x; i < (int64_t)B * L_out; i += blockDim.x) {
            const int b = (int)(i / L_out), l = (int)(i - (int64_t)b * L_out);
            s = __fadd_rn(s, ld_f32(gout + ((int64_t)b * C_out + co) * L_out + l));
        }
    }
    part[threadIdx.x] = s;
    __syncthreads();
    for (int w = 128; w > 0; w >>= 1) {
        if ((int)threadIdx.x < w)
            part[threadIdx.x] = __fadd_rn(part[threadIdx.x], part[threadIdx.x + w]);
        __syncthreads();
    }
    if (threadIdx.x == 0)
        gbias[co] = from_f32<T>(part[0]);
}

template <class T>
__global__ void __launch_bounds__(256) write_out_kernel(const float *src, T *dst, int64_t n) {
    const int64_t stride = (int64_t)gridDim.x * blockDim.x;
    const int64_t i0 = (int64_t)blockIdx.x * blockDim.x + threadIdx.x;
    // four elements at a time (a 16-byte load) where both buffers are aligned for it
    if ((reinterpret_cast<uintptr_t>(src) & 15) == 0 &&
        (reinterpret_cast<uintptr_t>(dst) & (4 * sizeof(T) - 1)) == 0) {
        const int64_t n4 = n / 4;
        for (int64_t i = i0; i < n4; i += stride) {
            const float4 v = __ldg(reinterpret_cast<const float4 *>(src) + i);
            T o[4] = {from_f32<T>(v.x), from_f32<T>(v.y), from_f32<T>(v.z), from_f32<T>(v.w)};
            if constexpr (sizeof(T) == 2)
                *reinterpret_cast<uint2 *>(dst + 4 * i) = *reinterpret_cast<const uint2 *>(o);
            else
                *reinterpret_cast<float4 *>(dst + 4 * i) = *reinterpret_cast<const float4 *>(o);
        }
        for (int64_t i = 4 * n4 + i0; i < n; i += stride)   // the last n % 4 elements
            dst[i] = from_f32<T>(src[i]);
        return;
    }
    for (int64_t i = i0; i < n; i += stride)
        dst[i] = from_f32<T>(src[i]);
}

// dst[row][0 .. L) = src[row][0 .. L) for every row, dst rows ld elements apart (the rest
// of a dst row is not written: readers stop at L).
__global__ void __launch_bounds__(256) pad_rows_kernel(const float *src, float *dst, int64_t rows,
                                                       int L, int ld) {
    const int64_t n = rows * L;
    for (int64_t i = (int64_t)blockIdx.x * blockDim.x + threadIdx.x; i < n;
         i += (int64_t)gridDim.x * blockDim.x) {
        const int64_t r = i / L;
        dst[r * ld + (i - r * L)] = __ldg(src + i);
    }
}

size_t align256(size_t x) { return (x + 255) / 256 * 256; }

// Splits of the weight gradient's batch sum: the largest divisor of B that brings the
// grid to about two waves of the SMs (1: no split, the GEMM writes grad_weight itself).
int wgrad_splits(const Problem &P) {
    const int sms = sm_count() > 0 ? sm_count() : 148;
    const int64_t tiles = (int64_t)((P.cin_g * P.K + kBN - 1) / kBN) *
                          ((P.cout_g + kBM - 1) / kBM) * P.groups;
    int want = (int)((2 * sms + tiles - 1) / tiles);
    if (want > P.B)
        want = P.B;
    int S = 1;
    for (int d = 1; d <= want; ++d)
        if (P.B % d == 0)
            S = d;
    return S;
}

// The tensor-core GEMMs serve 16-bit problems whose K-major operands TMA can read: rows
// of grad_out and of the columns (L_out elements), of grad_out transposed (C_out) and of
// W transposed per group (C_out / groups) all multiples of 16 bytes.
bool tc_backward(const Problem &P, const BackwardGrads &G) {
    if (P.dtype != DCN1D_BF16 && P.dtype != DCN1D_F16)
        return false;
    if (P.L_out % 8 || P.C_out % 8 || P.cout_g % 8)
        return false;
    if ((reinterpret_cast<uintptr_t>(G.gout) & 15) || (reinterpret_cast<uintptr_t>(P.w) & 15))
        return false;
    const int64_t rows = (int64_t)P.B * (P.C_in * P.K > P.C_out ? P.C_in * P.K : P.C_out);
    return (int64_t)P.B * P.L_out < (1LL << 31) && rows < (1LL << 31);
}

// fp32 problems on the tensor cores (three TF32 products): the transposed grad_out and W
// rows (C_out, C_out / groups elements) must be multiples of 16 bytes; the columns and
// grad_out of the weight gradient are kept with rows padded to a multiple of 4.
bool tc32_backward(const Problem &P, const BackwardGrads &G) {
    if (P.dtype != DCN1D_F32)
        return false;
    if (P.C_out % 4 || P.cout_g % 4)
        return false;
    if ((reinterpret_cast<uintptr_t>(G.gout) & 15) || (reinterpret_cast<uintptr_t>(P.w) & 15))
        return false;
    const int64_t lp = (P.L_out + 3) / 4 * 4;
    const int64_t rows = (int64_t)P.B * (P.C_in * P.K > P.C_out ? P.C_in * P.K : P.C_out);
    return (int64_t)P.B * lp < (1LL << 31) && rows < (1LL << 31);
}

// Splits of the tensor-core weight-gradient GEMM's batch sum: the largest divisor of B
// that brings its 128 x N tiles to about one or two waves of the SMs.
int wgrad_splits_tc(const Problem &P) {
    const int sms = sm_count() > 0 ? sm_count() : 148;
    const int nt = P.cout_g <= 128 ? (P.cout_g <= 64 ? 64 : 128) : 256;
    const int64_t tiles = (int64_t)((P.cin_g * P.K + 127) / 128) * ((P.cout_g + nt - 1) / nt) *
                          P.groups;
    int want = (int)((2 * sms + tiles - 1) / tiles);
    if (want > P.B)
        want = P.B;
    int S = 1;
    for (int d = 1; d <= want; ++d)
        if (P.B % d == 0)
            S = d;
    return S;
}

struct WsLayout {
    size_t dcols, cols, gx, goff, gmask, wpart, total;   // byte offsets (SIZE_MAX: not used)
    size_t goutT, wT;    // tensor-core path: grad_out and W transposed (16-bit)
    int wsplits;
    bool tc;
    bool fused;          // tensor-core path whose column gradients stay on chip
    bool tc32;           // fp32 on the tensor cores (three TF32 products)
    int lp;              // row stride of the columns (and of goutP) in elements
    size_t goutP;        // tc32: grad_out with rows padded to lp (fp32)
};

WsLayout ws_layout(const Problem &P, const BackwardGrads &G) {
    WsLayout w;
    w.tc = tc_backward(P, G);
    const size_t ncol = (size_t)P.B * P.C_in * P.K * P.L_out * 4;
    const size_t noff = (size_t)P.B * P.offset_groups * P.L_out * P.K * 4;
    const bool need_dcols = G.x || G.off || G.mask;
    w.fused = w.tc && need_dcols && gemm_sample_supported(P);
    w.tc32 = !w.tc && tc32_backward(P, G);
    w.lp = w.tc32 ? (P.L_out + 3) / 4 * 4 : P.L_out;
    const size_t ncolp = (size_t)P.B * P.C_in * P.K * w.lp * 4;
    const size_t tsz = w.tc32 ? 4 : 2;   // element size of the transposed copies
    size_t at = 0;
    w.dcols = (need_dcols && !w.fused) ? at : SIZE_MAX;
    at += (need_dcols && !w.fused) ? align256(ncol) : 0;
    w.cols = G.w ? at : SIZE_MAX;   // the 16-bit tensor-core path keeps them in 16 bits
    at += G.w ? align256(w.tc ? ncol / 2 : ncolp) : 0;
    const bool tr = (w.tc || w.tc32) && need_dcols;
    w.goutT = tr ? at : SIZE_MAX;
    at += tr ? align256((size_t)P.B * P.C_out * P.L_out * tsz) : 0;
    w.wT = tr ? at : SIZE_MAX;
    at += tr ? align256((size_t)P.C_out * P.cin_g * P.K * tsz) : 0;
    w.goutP = (w.tc32 && G.w) ? at : SIZE_MAX;
    at += (w.tc32 && G.w) ? align256((size_t)P.B * P.C_out * w.lp * 4) : 0;
    w.gx = G.x ? at : SIZE_MAX;
    at += G.x ? align256((size_t)P.B * P.C_in * P.L_in * 4) : 0;
    w.goff = G.off ? at : SIZE_MAX;
    at += G.off ? align256(noff) : 0;
    w.gmask = G.mask ? at : SIZE_MAX;
    at += G.mask ? align256(noff) : 0;
    w.wsplits = G.w ? ((w.tc || w.tc32) ? wgrad_splits_tc(P) : wgrad_splits(P)) : 1;
    // the tensor-core GEMMs write fp32 slices even unsplit (then converted)
    const bool parts = G.w && (w.wsplits > 1 || w.tc || w.tc32);
    w.wpart = parts ? at : SIZE_MAX;
    at += parts ? align256((size_t)w.wsplits * P.C_out * P.cin_g * P.K * 4) : 0;
    w.total = at;
    return w;
}

unsigned grid_1d(int64_t n) {
    const int64_t want = (n + 255) / 256;
    return (unsigned)(want < 65535LL * 16 ? want : 65535LL * 16);
}

template <class T>
cudaError_t run_backward(const Problem &P, const BackwardGrads &G, void *ws, cudaStream_t s,
                         int *launches) {
    const WsLayout L = ws_layout(P, G);
    unsigned char *wsb = static_cast<unsigned char *>(ws);
    float *dcols = L.dcols != SIZE_MAX ? reinterpret_cast<float *>(wsb + L.dcols) : nullptr;
    float *cols = (L.cols != SIZE_MAX && !L.tc) ? reinterpret_cast<float *>(wsb + L.cols)
                                                : nullptr;
    T *cols16 = (L.cols != SIZE_MAX && L.tc) ? reinterpret_cast<T *>(wsb + L.cols) : nullptr;
    T *goutT = L.goutT != SIZE_MAX ? reinterpret_cast<T *>(wsb + L.goutT) : nullptr;
    T *wT = L.wT != SIZE_MAX ? reinterpret_cast<T *>(wsb + L.wT) : nullptr;
    float *goutP = L.goutP != SIZE_MAX ? reinterpret_cast<float *>(wsb + L.goutP) : nullptr;
    float *gx = L.gx != SIZE_MAX ? reinterpret_cast<float *>(wsb + L.gx) : nullptr;
    float *goff = L.goff != SIZE_MAX ? reinterpret_cast<float *>(wsb + L.goff) : nullptr;
    float *gmask = L.gmask != SIZE_MAX ? reinterpret_cast<float *>(wsb + L.gmask) : nullptr;
    float *wpart = L.wpart != SIZE_MAX ? reinterpret_cast<float *>(wsb + L.wpart) : nullptr;
    const T *w = static_cast<const T *>(P.w);
    const T *gout = static_cast<const T *>(G.gout);
    const int Kg = P.cin_g * P.K;
    const bool want_dcols = G.x || G.off || G.mask;   // (scratch pointers are NULL when
    const bool want_cols = G.w != nullptr;           //  their size is zero)
    cudaError_t e;
    int n = 0;
    const int64_t nx = (int64_t)P.B * P.C_in * P.L_in;
    const int64_t noff = (int64_t)P.B * P.offset_groups * P.L_out * P.K;
    if (gx && (e = cudaMemsetAsync(gx, 0, nx * 4, s)) != cudaSuccess)
        return e;
    if (goff && (e = cudaMemsetAsync(goff, 0, noff * 4, s)) != cudaSuccess)
        return e;
    if (gmask && (e = cudaMemsetAsync(gmask, 0, noff * 4, s)) != cudaSuccess)
        return e;

    if (want_dcols && P.B > 0 && L.tc) {
        // 1. on the tensor cores: D[l][m] = sum_co goutT[b][l][g*cout_g + co] * wT[g][m][co],
        // stored to dcols[b][g*Kg + m][l] (lanes = consecutive l)
        const dim3 tb(256);
        transpose_kernel<T><<<dim3((P.L_out + 31) / 32, (P.C_out + 31) / 32, P.B), tb, 0, s>>>(
            gout, goutT, P.C_out, P.L_out, P.L_out, P.C_out, (int64_t)P.C_out * P.L_out,
            (int64_t)P.L_out * P.C_out);
        transpose_kernel<T><<<dim3((Kg + 31) / 32, (P.cout_g + 31) / 32, P.groups), tb, 0, s>>>(
            w, wT, P.cout_g, Kg, Kg, P.cout_g, (int64_t)P.cout_g * Kg, (int64_t)Kg * P.cout_g);
        if ((e = cudaGetLastError()) != cudaSuccess)
            return e;
        n += 2;
        for (int gi = 0; L.fused && gi < P.groups; ++gi) {
            // the column gradient's GEMM with the sampling gradient as its drain (the
            // sampled columns too, when the weight gradient is wanted)
            if ((e = launch_gemm_sample(P, gi, goutT + (int64_t)gi * P.cout_g,
                                        wT + (int64_t)gi * Kg * P.cout_g,
                                        want_cols ? cols16 : nullptr, gx, goff, gmask, s)) !=
                cudaSuccess)
                return e;
            ++n;
        }
        for (int gi = 0; !L.fused && gi < P.groups; ++gi) {
            if ((e = launch_gemm_tc(P.dtype, goutT + (int64_t)gi * P.cout_g,
                                    (int64_t)P.B * P.L_out, P.C_out, 0, P.L_out, 0,
                                    wT + (int64_t)gi * Kg * P.cout_g, Kg, P.cout_g, 0, 0, 0,
                                    P.L_out, Kg, P.cout_g, 1, P.B,
                                    dcols + (int64_t)gi * Kg * P.L_out, 1, P.L_out,
                                    (int64_t)P.C_in * P.K * P.L_out, s)) != cudaSuccess)
                return e;
            ++n;
        }
    } else if (want_dcols && P.B > 0 && L.tc32) {
        // 1. fp32 on the tensor cores, three TF32 products: D[n][m] = sum_co goutT[n][g*cout_g
        // + co] * wT[g][m][co] over the flattened rows n = b * L_out + l, stored to
        // dcols[b][g*Kg + m][l]
        const dim3 tb(256);
        transpose_kernel<T><<<dim3((P.L_out + 31) / 32, (P.C_out + 31) / 32, P.B), tb, 0, s>>>(
            gout, goutT, P.C_out, P.L_out, P.L_out, P.C_out, (int64_t)P.C_out * P.L_out,
            (int64_t)P.L_out * P.C_out);
        transpose_kernel<T><<<dim3((Kg + 31) / 32, (P.cout_g + 31) / 32, P.groups), tb, 0, s>>>(
            w, wT, P.cout_g, Kg, Kg, P.cout_g, (int64_t)P.cout_g * Kg, (int64_t)Kg * P.cout_g);
        if ((e = cudaGetLastError()) != cudaSuccess)
            return e;
        n += 2;
        for (int gi = 0; gi < P.groups; ++gi) {
            if ((e = launch_gemm_x3(reinterpret_cast<const float *>(goutT) + (int64_t)gi * P.cout_g,
                                    (int64_t)P.B * P.L_out, P.C_out, 0, 0, 0,
                                    reinterpret_cast<const float *>(wT) +
                                        (int64_t)gi * Kg * P.cout_g,
                                    Kg, P.cout_g, 0, 0, 0, P.L_out, Kg, P.cout_g, 1, P.B, P.L_out,
                                    dcols + (int64_t)gi * Kg * P.L_out, 1, P.L_out,
                                    (int64_t)P.C_in * P.K * P.L_out, s)) != cudaSuccess)
                return e;
            ++n;
        }
    } else if (want_dcols && P.B > 0) {
        // 1. dcols[b][g*Kg + m][l] = sum_co W[g*cout_g + co][m] * gout[b][g*cout_g + co][l]
        GemmArgs g;
        memset(&g, 0, sizeof(g));
        g.M = Kg;
        g.N = P.L_out;
        g.Kd = P.cout_g;
        g.R = 1;
        g.ng = P.groups;
        g.a_sm = 1;
        g.a_sk = Kg;
        g.a_sg = (int64_t)P.cout_g * Kg;
        g.b_sk = P.L_out;
        g.b_sn = 1;
        g.b_sb = (int64_t)P.C_out * P.L_out;
        g.b_sg = (int64_t)P.cout_g * P.L_out;
        g.c_sm = P.L_out;
        g.c_sn = 1;
        g.c_sb = (int64_t)P.C_in * P.K * P.L_out;
        g.c_sg = (int64_t)Kg * P.L_out;
        if ((e = run_gemm<T, T, float, true, true>(w, gout, dcols, g, P.B * P.groups, s)) !=
            cudaSuccess)
            return e;
        ++n;
    }
    if ((want_dcols && !L.fused) || (want_cols && !(L.fused && want_dcols))) {
        // 2. sampling gradient and sampled columns (the fused path did both already)
        SampArgs a;
        memset(&a, 0, sizeof(a));
        a.P = P;
        a.cols_ld = L.lp;
        a.nchunk = (P.cin_per_og + kChunk - 1) / kChunk;
        a.nlb = (P.L_out + kSgRows - 1) / kSgRows;
        // grad_x window: the receptive fields of a block's positions, plus a margin for
        // unconstrained taps; past 48 KB of shared memory, global atomics only
        a.margin = P.unconstrained ? 16 : 0;
        {
            const int64_t w = (int64_t)(kSgRows - 1) * P.stride +
                              (int64_t)P.dilation * (P.K - 1) + 2 + 2 * a.margin;
            a.win = (w * kChunk * 4 <= 48 * 1024) ? (int)w : 0;
        }
        a.dcols = dcols;
        a.cols = cols;
        a.cols16 = cols16;
        a.gx = gx;
        a.goff = goff;
        a.gmask = gmask;
        const int64_t nt = (int64_t)P.B * a.nchunk * P.offset_groups * P.L_out;
        const int64_t blocks = (int64_t)P.B * P.offset_groups * a.nchunk * a.nlb;
        const size_t shm = (gx && dcols) ? (size_t)a.win * kChunk * 4 : 0;
        if (nt == 0) {
            // empty batch: no columns, no sampling gradient
        } else if (blocks >= (1LL << 31)) {
            return cudaErrorInvalidValue;
        } else if (P.mask)
            sample_grad_kernel<T, true><<<(unsigned)blocks, kSgRows, shm, s>>>(a);
        else
            sample_grad_kernel<T, false><<<(unsigned)blocks, kSgRows, shm, s>>>(a);
        if ((e = cudaGetLastError()) != cudaSuccess)
            return e;
        n += nt > 0;
    }
    if (want_cols && L.tc) {
        // 3. on the tensor cores, per split z of the batch sum: D[m][co] = sum over the
        // split's batches b and l of cols16[b][g*Kg + m][l] * gout[b][g*cout_g + co][l],
        // stored to wpart[z][g*cout_g + co][m]; then the slices added in split order
        const int S = L.wsplits, rps = P.B / S;
        if (P.B > 0) {
            for (int gi = 0; gi < P.groups; ++gi) {
                if ((e = launch_gemm_tc(P.dtype, cols16, (int64_t)P.B * P.C_in * P.K, P.L_out,
                                        gi * Kg, rps * P.C_in * P.K, P.C_in * P.K, gout,
                                        (int64_t)P.B * P.C_out, P.L_out, gi * P.cout_g,
                                        rps * P.C_out, P.C_out, Kg, P.cout_g, P.L_out, rps, S,
                                        wpart + (int64_t)gi * P.cout_g * Kg, 1, Kg,
                                        (int64_t)P.C_out * Kg, s)) != cudaSuccess)
                    return e;
                ++n;
            }
        }
        const int64_t nw = (int64_t)P.C_out * Kg;
        if (P.B > 0)
            sum_splits_kernel<T><<<grid_1d(nw), 256, 0, s>>>(wpart, static_cast<T *>(G.w), S, nw);
        else if ((e = cudaMemsetAsync(G.w, 0, nw * sizeof(T), s)) != cudaSuccess)
            return e;
        if ((e = cudaGetLastError()) != cudaSuccess)
            return e;
        n += P.B > 0;
    } else if (want_cols && L.tc32) {
        // 3. fp32 on the tensor cores, as the 16-bit form above, with grad_out and the
        // columns in rows padded to lp elements (TMA rows are multiples of 16 bytes)
        const int S = L.wsplits, rps = P.B / S;
        const int64_t nw = (int64_t)P.C_out * Kg;
        if (P.B > 0) {
            pad_rows_kernel<<<grid_1d((int64_t)P.B * P.C_out * P.L_out), 256, 0, s>>>(
                reinterpret_cast<const float *>(gout), goutP, (int64_t)P.B * P.C_out, P.L_out,
                L.lp);
            if ((e = cudaGetLastError()) != cudaSuccess)
                return e;
            ++n;
            for (int gi = 0; gi < P.groups; ++gi) {
                if ((e = launch_gemm_x3(cols, (int64_t)P.B * P.C_in * P.K, L.lp, gi * Kg,
                                        rps * P.C_in * P.K, P.C_in * P.K, goutP,
                                        (int64_t)P.B * P.C_out, L.lp, gi * P.cout_g,
                                        rps * P.C_out, P.C_out, Kg, P.cout_g, P.L_out, rps, S, 0,
                                        wpart + (int64_t)gi * P.cout_g * Kg, 1, Kg,
                                        (int64_t)P.C_out * Kg, s)) != cudaSuccess)
                    return e;
                ++n;
            }
            sum_splits_kernel<T><<<grid_1d(nw), 256, 0, s>>>(wpart, static_cast<T *>(G.w), S, nw);
            if ((e = cudaGetLastError()) != cudaSuccess)
                return e;
            ++n;
        } else if ((e = cudaMemsetAsync(G.w, 0, nw * sizeof(T), s)) != cudaSuccess) {
            return e;
        }
    } else if (want_cols) {
        // 3. gW[g*cout_g + co][m] = sum_b sum_l gout[b][g*cout_g + co][l] * cols[b][g*Kg + m][l]
        // (zeros for an empty batch).  Split s of the batch sum covers batches
        // [s * rps, (s + 1) * rps) (blockIdx.z = s * groups + group) and writes its own
        // fp32 slice; the slices are then added in split order.
        const int S = L.wsplits, rps = S > 1 ? P.B / S : P.B;
        GemmArgs g;
        memset(&g, 0, sizeof(g));
        g.M = P.cout_g;
        g.N = Kg;
        g.Kd = P.L_out;
        g.R = rps;
        g.ng = P.groups;
        g.a_sm = P.L_out;
        g.a_sk = 1;
        g.a_sg = (int64_t)P.cout_g * P.L_out;
        g.a_sr = (int64_t)P.C_out * P.L_out;
        g.a_sb = g.a_sr * rps;
        g.b_sk = 1;
        g.b_sn = P.L_out;
        g.b_sg = (int64_t)Kg * P.L_out;
        g.b_sr = (int64_t)P.C_in * P.K * P.L_out;
        g.b_sb = g.b_sr * rps;
        g.c_sm = Kg;
        g.c_sn = 1;
        g.c_sg = (int64_t)P.cout_g * Kg;
        g.c_sb = (int64_t)P.C_out * Kg;
        if (S > 1) {
            if ((e = run_gemm<T, float, float, false, false>(gout, cols, wpart, g, S * P.groups,
                                                             s)) != cudaSuccess)
                return e;
            const int64_t nw = (int64_t)P.C_out * Kg;
            sum_splits_kernel<T><<<grid_1d(nw), 256, 0, s>>>(wpart, static_cast<T *>(G.w), S, nw);
            if ((e = cudaGetLastError()) != cudaSuccess)
                return e;
            n += 2;
        } else {
            if ((e = run_gemm<T, float, T, false, false>(gout, cols, static_cast<T *>(G.w), g,
                                                           P.groups, s)) != cudaSuccess)
                return e;
            ++n;
        }
    }
    if (G.bias) {   // 4.
        bias_grad_kernel<T><<<P.C_out, 256, 0, s>>>(gout, static_cast<T *>(G.bias), P.B, P.C_out,
                                                    P.L_out);
        if ((e = cudaGetLastError()) != cudaSuccess)
            return e;
        ++n;
    }
    // 5. scratch -> outputs in the input type
    if (gx && nx > 0) {
        write_out_kernel<T><<<grid_1d(nx), 256, 0, s>>>(gx, static_cast<T *>(G.x), nx);
        ++n;
    }
    if (goff && noff > 0) {
        write_out_kernel<T><<<grid_1d(noff), 256, 0, s>>>(goff, static_cast<T *>(G.off), noff);
        ++n;
    }
    if (gmask && noff > 0) {
        write_out_kernel<T><<<grid_1d(noff), 256, 0, s>>>(gmask, static_cast<T *>(G.mask), noff);
        ++n;
    }
    *launches = n;
    return cudaGetLastError();
}

}  // namespace

size_t backward_workspace(const Problem &P, const BackwardGrads &G) {
    return ws_layout(P, G).total;
}

bool backward_uses_tensor_cores(const Problem &P, const BackwardGrads &G) {
    return tc_backward(P, G) || tc32_backward(P, G);
}

cudaError_t launch_backward(const Problem &P, const BackwardGrads &G, void *workspace,
                            cudaStream_t stream, int *launches) {
    *launches = 0;
    if (P.dtype == DCN1D_BF16)
        return run_backward<__nv_bfloat16>(P, G, workspace, stream, launches);
    if (P.dtype == DCN1D_F16)
        return run_backward<__half>(P, G, workspace, stream, launches);
    return run_backward<float>(P, G, workspace, stream, launches);
}

}  // namespace dcn1d
