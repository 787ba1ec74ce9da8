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
//  * A task is 32 consecutive output pixels (flattened n, oy, ox) x FB
//    filters; lane <-> pixel, so each epilogue store of a warp is 32
//    consecutive NCHW elements (128 contiguous bytes).  The lane gathers its
//    pixel's 9 taps x CW words into registers from the packed input (L1/L2
//    resident: the packed input is 1/16 the size of the bf16 one).  A tap
//    outside the image is the all-zero word, i.e. +1 (zero-padded real input,
//    then sign).
//  * For each filter: XOR over 9*CW words for each of the P pixels, counted
//    with the carry-save 7:3 counter of the GEMM (4 POPC per 8 words), then
//    the epilogue for that (pixel, filter) with alpha/gamma/beta read from
//    shared memory.
//  * The grid is a whole number of CTAs per SM; each CTA owns a contiguous,
//    equal share of the tasks and its warps take them one at a time from a
//    shared-memory counter, so the work per SM is balanced to one task.
#pragma once

#include "common.cuh"
#include "gemm_popc.cuh"   // popc8_csa

namespace bnn {
namespace conv {
constexpr int THREADS = 256;
constexpr int WARPS = THREADS / 32;
constexpr int FB = 16;          // filters per task
constexpr int CTAS_PER_SM = 4;
}  // namespace conv

struct ConvEpilogue {
    int mode;             // BNN_OUT_INT32, BNN_OUT_SCALED_F32, BNN_OUT_AFFINE_F32
    const float* alpha;
    const float* gamma;
    const float* beta;
    void* out;            // NCHW
};

// popcount of the XOR of two n-word strings: groups of 8 words go through the
// carry-save 7:3 counter (4 POPC per 8 words), the rest through plain POPC.
template <int NW>
__device__ __forceinline__ uint32_t xor_popc_words(const uint32_t* a, const uint32_t* w) {
    uint32_t d = 0;
    #pragma unroll
    for (int g = 0; g + 8 <= NW; g += 8) {
        uint32_t x[8];
        #pragma unroll
        for (int k = 0; k < 8; ++k) x[k] = a[g + k] ^ w[g + k];
        d = popc8_csa_acc(x, d);
    }
    #pragma unroll
    for (int k = NW / 8 * 8; k < NW; ++k) d += __popc(a[k] ^ w[k]);
    return d;
}

template <int CW>
__global__ void __launch_bounds__(conv::THREADS, conv::CTAS_PER_SM)
xnor_conv3x3_kernel(const uint32_t* __restrict__ X, int n, int c, int h, int w,
                    const uint32_t* __restrict__ Wp, int64_t ldw, int cout, int stride, int pad,
                    int oh, int ow, ConvEpilogue ep) {
    using namespace conv;
    constexpr int KW = 9 * CW;                 // words per filter row
    constexpr int KWP = (KW + 3) / 4 * 4;      // padded to 16 bytes in shared memory
    extern __shared__ __align__(16) uint32_t ws[];
    __shared__ unsigned long long next_task;
    float* par = reinterpret_cast<float*>(ws + cout * KWP);   // alpha, gamma, beta per filter
    for (int i = threadIdx.x; i < cout * KWP; i += THREADS) {
        const int co = i / KWP, k = i % KWP;
        ws[i] = (k < KW) ? Wp[(int64_t)co * ldw + k] : 0u;
    }
    for (int co = threadIdx.x; co < cout; co += THREADS) {
        par[co] = ep.mode != BNN_OUT_INT32 ? ep.alpha[co] : 0.0f;
        par[cout + co] = ep.mode == BNN_OUT_AFFINE_F32 ? ep.gamma[co] : 0.0f;
        par[2 * cout + co] = ep.mode == BNN_OUT_AFFINE_F32 ? ep.beta[co] : 0.0f;
    }
    const int64_t plane = (int64_t)oh * ow;
    const int64_t npix = (int64_t)n * plane;
    const int fblocks = (cout + FB - 1) / FB;
    const int64_t tasks = (npix + 31) / 32 * fblocks;
    // This CTA's contiguous share of the tasks (equal to within one task).
    const int64_t t_begin = tasks * blockIdx.x / gridDim.x;
    const int64_t t_end = tasks * (blockIdx.x + 1) / gridDim.x;
    if (threadIdx.x == 0) next_task = (unsigned long long)t_begin;
    __syncthreads();

    const int lane = threadIdx.x & 31;
    const int Ktrue = 9 * c;
    while (true) {
        unsigned long long tk = 0;
        if (lane == 0) tk = atomicAdd(&next_task, 1ull);
        const int64_t task = (int64_t)__shfl_sync(0xffffffffu, tk, 0);
        if (task >= t_end) break;
        const int64_t pblock = task / fblocks;
        const int co0 = (int)(task % fblocks) * FB;
        const int64_t q = pblock * 32 + lane;          // this lane's output pixel
        uint32_t a[KW];
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
            for (int j = 0; j < CW; ++j) a[t * CW + j] = in ? __ldg(X + off + j) : 0u;
        }
        const int64_t obase = b * cout * plane + (q < npix ? q % plane : 0);
        const int co_end = min(co0 + FB, cout);
        for (int co = co0; co < co_end; ++co) {
            uint32_t wr[KW];
            #pragma unroll
            for (int k4 = 0; k4 < KWP; k4 += 4) {
                const uint4 wv = *reinterpret_cast<const uint4*>(ws + co * KWP + k4);
                if (k4 + 0 < KW) wr[k4 + 0] = wv.x;
                if (k4 + 1 < KW) wr[k4 + 1] = wv.y;
                if (k4 + 2 < KW) wr[k4 + 2] = wv.z;
                if (k4 + 3 < KW) wr[k4 + 3] = wv.w;
            }
            const uint32_t d = xor_popc_words<KW>(a, wr);
            if (q >= npix) continue;
            const int64_t o = obase + (int64_t)co * plane;
            const int32_t sv = Ktrue - 2 * (int32_t)d;
            if (ep.mode == BNN_OUT_INT32) {
                static_cast<int32_t*>(ep.out)[o] = sv;
            } else {
                float y = par[co] * (float)sv;
                if (ep.mode == BNN_OUT_AFFINE_F32) y = fmaf(par[cout + co], y, par[2 * cout + co]);
                static_cast<float*>(ep.out)[o] = y;
            }
        }
    }
}

}  // namespace bnn
