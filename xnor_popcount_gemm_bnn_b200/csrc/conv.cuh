// Binary 3x3 convolution as an implicit GEMM over packed per-pixel channel
// words: M = n*oh*ow output pixels, N = cout filters, K = 9*c binary elements.
//
// "Extreme Quantization: Binary, Ternary & 1-bit LLMs", eq. (4) and (6);
// eq. (1) with one alpha per filter ("Binary Neural Network (BNN)" glossary:
// scaling factors for each weight filter); the affine epilogue carries the
// BatchNorm scale and shift of that glossary paragraph.
//
// Design (sm_100a):
//  * The packed filters (cout x 9*CW words, a few KB) are staged once per CTA
//    in shared memory; every lane of a warp reads the same filter word, so
//    those reads are broadcasts.
//  * Lane <-> output pixel in flattened (n, oy, ox) order, so each epilogue
//    store of a warp is 32 consecutive NCHW elements (128 contiguous bytes).
//    Each lane owns P pixels (p, p + 32, ...) and gathers their 9 taps x CW
//    words into registers from the packed input (L1/L2 resident: the packed
//    input is 1/16 the size of the bf16 one).  A tap outside the image is the
//    all-zero word, i.e. +1 (zero-padded real input, then sign).
//  * For each filter: XOR + POPC over 9*CW words for each of the P pixels,
//    then the epilogue for that (pixel, filter).
#pragma once

#include "common.cuh"

namespace bnn {
namespace conv {
constexpr int THREADS = 256;
constexpr int WARPS = THREADS / 32;
constexpr int P = 2;   // pixels per lane
}  // namespace conv

struct ConvEpilogue {
    int mode;             // BNN_OUT_INT32, BNN_OUT_SCALED_F32, BNN_OUT_AFFINE_F32
    const float* alpha;
    const float* gamma;
    const float* beta;
    void* out;            // NCHW
};

template <int CW>
__global__ void __launch_bounds__(conv::THREADS)
xnor_conv3x3_kernel(const uint32_t* __restrict__ X, int n, int c, int h, int w,
                    const uint32_t* __restrict__ Wp, int64_t ldw, int cout, int stride, int pad,
                    int oh, int ow, ConvEpilogue ep) {
    using namespace conv;
    constexpr int KW = 9 * CW;                 // words per filter row
    constexpr int KWP = (KW + 3) / 4 * 4;      // padded to 16 bytes in shared memory
    extern __shared__ __align__(16) uint32_t ws[];
    for (int i = threadIdx.x; i < cout * KWP; i += THREADS) {
        const int co = i / KWP, k = i % KWP;
        ws[i] = (k < KW) ? Wp[(int64_t)co * ldw + k] : 0u;
    }
    __syncthreads();

    const int warp = threadIdx.x >> 5;
    const int lane = threadIdx.x & 31;
    const int64_t plane = (int64_t)oh * ow;
    const int64_t npix = (int64_t)n * plane;
    const int64_t base = ((int64_t)blockIdx.x * WARPS + warp) * (32 * P);
    const int Ktrue = 9 * c;

    uint32_t a[P][KW];
    int64_t pix[P];
    #pragma unroll
    for (int pp = 0; pp < P; ++pp) {
        const int64_t q = base + lane + 32 * pp;
        pix[pp] = q;
        int64_t b = 0, oy = 0, ox = 0;
        if (q < npix) {
            b = q / plane;
            const int64_t r = q % plane;
            oy = r / ow;
            ox = r % ow;
        }
        #pragma unroll
        for (int t = 0; t < 9; ++t) {
            const int iy = (int)oy * stride - pad + t / 3;
            const int ix = (int)ox * stride - pad + t % 3;
            const bool in = q < npix && iy >= 0 && iy < h && ix >= 0 && ix < w;
            // Offset 0 for taps outside the image, so no out-of-range address is formed.
            const int64_t off = in ? ((b * h + iy) * (int64_t)w + ix) * CW : 0;
            #pragma unroll
            for (int j = 0; j < CW; ++j) a[pp][t * CW + j] = in ? __ldg(X + off + j) : 0u;
        }
    }

    for (int co = 0; co < cout; ++co) {
        const uint32_t* wr = ws + co * KWP;
        uint32_t d[P];
        #pragma unroll
        for (int pp = 0; pp < P; ++pp) d[pp] = 0u;
        #pragma unroll
        for (int k4 = 0; k4 < KWP; k4 += 4) {
            const uint4 wv = *reinterpret_cast<const uint4*>(wr + k4);
            const uint32_t wk[4] = {wv.x, wv.y, wv.z, wv.w};
            #pragma unroll
            for (int e = 0; e < 4; ++e) {
                if (k4 + e < KW) {
                    #pragma unroll
                    for (int pp = 0; pp < P; ++pp) d[pp] += __popc(a[pp][k4 + e] ^ wk[e]);
                }
            }
        }
        float al = 0.f, ga = 0.f, be = 0.f;
        if (ep.mode != BNN_OUT_INT32) al = ep.alpha[co];
        if (ep.mode == BNN_OUT_AFFINE_F32) { ga = ep.gamma[co]; be = ep.beta[co]; }
        #pragma unroll
        for (int pp = 0; pp < P; ++pp) {
            const int64_t q = pix[pp];
            if (q >= npix) continue;
            const int64_t b = q / plane, r = q % plane;
            const int64_t o = (b * cout + co) * plane + r;
            const int32_t s = Ktrue - 2 * (int32_t)d[pp];
            if (ep.mode == BNN_OUT_INT32) {
                static_cast<int32_t*>(ep.out)[o] = s;
            } else {
                float y = al * (float)s;
                if (ep.mode == BNN_OUT_AFFINE_F32) y = fmaf(ga, y, be);
                static_cast<float*>(ep.out)[o] = y;
            }
        }
    }
}

}  // namespace bnn
