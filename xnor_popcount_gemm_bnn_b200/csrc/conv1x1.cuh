// Binary 1x1 convolution with stride (the downsampling projection of a
// ResNet-class block) as a GEMM over packed per-pixel channel words:
// M = n*oh*ow output pixels, N = cout filters, K = c binary elements.
//
// "Extreme Quantization: Binary, Ternary & 1-bit LLMs", eq. (4) and (6), with
// eq. (1) (one alpha per filter) and the affine epilogue of the 3x3 kernel;
// the vision workload of "Perfected Concept: Extreme Low-Bit Inference"
// (edge vision BNNs) and the ResNet-class rows of "State of the Art Survey
// (2016 -> 2026)".
//
// A lane owns P pixels of a block of 32P consecutive output pixels (P = 2 up
// to 256 channels), lane l taking pixels l, l+32, ... (each warp store is
// 128 contiguous NCHW bytes); a filter's words are read from shared memory
// once for the lane's P pixels.  A lane loads each of
// its pixels' cw words once (input pixel (s*oy, s*ox)); CWP >= cw (1, 2, 4, 8
// or 16) is the compile-time capacity, words past cw are 0 on both sides.  With c <= 512 channels the
// row is at most 16 words, so the kernel is bound by its fp32 NCHW output
// stream.
#pragma once

#include <type_traits>

#include "conv.cuh"

namespace bnn {

namespace c1x1 {
// Output pixels per lane (a pixel block is 32 * P pixels): 2, or 1 for rows
// of 16 words.
__host__ __device__ constexpr int pixels_per_lane(int cwp) { return cwp <= 8 ? 2 : 1; }
}  // namespace c1x1

// MODE: BNN_OUT_INT32, BNN_OUT_SCALED_F32 or BNN_OUT_AFFINE_F32 (the epilogue
// is compiled per mode).  y = fma(ga_co, s, be_co) with ga = alpha (SCALED) or
// fp32(gamma * alpha) (AFFINE) and be = 0 or beta, staged once per CTA.
// Pixel indices are 32-bit (n*oh*ow and cout*oh*ow below 2^31, checked by
// the launcher).
//
// Work split: the units (pixel block, filter), pixel-block major, are cut
// into one contiguous, equal (to one unit) run per warp of the grid.  A warp
// gathers a pixel block's input words once and then walks that block's
// filters of its run, so the load balance is one unit and the gather is
// repeated only where a run crosses a block boundary.
template <int CWP, int MODE>
__global__ void __launch_bounds__(conv::THREADS, conv::CTAS_PER_SM)
xnor_conv1x1_kernel(const uint32_t* __restrict__ X, int n, int c, int h, int w, const uint32_t* __restrict__ Wp,
                    int64_t ldw, int cout, int stride, int oh, int ow, ConvEpilogue ep) {
    using namespace conv;
    constexpr int P = c1x1::pixels_per_lane(CWP);
    constexpr int KWP = (CWP + 3) / 4 * 4;     // filter row in shared memory, 16-byte multiple
    using OutT = typename std::conditional<MODE == BNN_OUT_INT32, int32_t, float>::type;
    extern __shared__ __align__(16) uint32_t ws1[];
    const int cw = (c + 31) / 32;
    float* ga = reinterpret_cast<float*>(ws1 + cout * KWP);
    float* be = ga + cout;
    // Programmatic dependent launch: the next launch may be scheduled once
    // every CTA of this grid has started (its CTAs then take SMs as these
    // exit); every read of memory the previous kernel may write (filters,
    // parameters, input) and every store follow the wait for that kernel.
    grid_dependents_launch();
    grid_dependency_wait();
    for (int i = threadIdx.x; i < cout * KWP; i += THREADS) {
        const int co = i / KWP, k = i % KWP;
        ws1[i] = (k < cw) ? Wp[(int64_t)co * ldw + k] : 0u;
    }
    for (int co = threadIdx.x; co < cout; co += THREADS) {
        if constexpr (MODE == BNN_OUT_SCALED_F32) {
            ga[co] = ep.alpha[co];
            be[co] = 0.0f;
        } else if constexpr (MODE == BNN_OUT_AFFINE_F32) {
            ga[co] = ep.gamma[co] * ep.alpha[co];
            be[co] = ep.beta[co];
        }
    }
    __syncthreads();
    const int plane = oh * ow;
    const int npix = n * plane;
    const int npb = (npix + 32 * P - 1) / (32 * P);
    const int lane = threadIdx.x & 31;
    const int64_t gw = (int64_t)blockIdx.x * WARPS + (threadIdx.x >> 5);
    const int64_t nwarps = (int64_t)gridDim.x * WARPS;
    const int64_t units = (int64_t)npb * cout;
    int64_t u = units * gw / nwarps;
    const int64_t u_end = units * (gw + 1) / nwarps;
    OutT* out = static_cast<OutT*>(ep.out);
    while (u < u_end) {
        const int pb = (int)(u / cout);
        const int co_begin = (int)(u - (int64_t)pb * cout);
        const int co_stop = (int)min((int64_t)cout, u_end - (int64_t)pb * cout);
        // Lane pixels q_p = pb*32P + 32p + lane: each store of a warp is 32
        // consecutive pixels of one output plane (unless a plane ends inside).
        uint32_t a[P][CWP];
        OutT* op[P];
        bool ok[P];
        #pragma unroll
        for (int p = 0; p < P; ++p) {
            const int q = pb * (32 * P) + 32 * p + lane;
            ok[p] = q < npix;
            const int b = ok[p] ? q / plane : 0;
            const int r = ok[p] ? q - b * plane : 0;
            const int oy = r / ow, ox = r - (r / ow) * ow;
            const int64_t off = (((int64_t)b * h + (int64_t)oy * stride) * w + (int64_t)ox * stride) * cw;
            #pragma unroll
            for (int j = 0; j < CWP; ++j) a[p][j] = (ok[p] && j < cw) ? __ldg(X + off + j) : 0u;
            op[p] = out + ((int64_t)b * cout * plane + r);
        }
        for (int co = co_begin; co < co_stop; ++co) {
            uint32_t wr[CWP];
            #pragma unroll
            for (int k = 0; k < CWP; ++k) wr[k] = ws1[co * KWP + k];
            float g = 0.0f, bb = 0.0f;
            if constexpr (MODE != BNN_OUT_INT32) {
                g = ga[co];
                bb = be[co];
            }
            const int co_off = co * plane;
            #pragma unroll
            for (int p = 0; p < P; ++p) {
                const uint32_t d = xor_popc_words<CWP>(a[p], wr);
                const int32_t sv = c - 2 * (int32_t)d;
                if (!ok[p]) continue;
                if constexpr (MODE == BNN_OUT_INT32) {
                    op[p][co_off] = sv;
                } else {
                    // float(sv) without the conversion unit: 0x4B400000 is the
                    // float 1.5 * 2^23, whose unit in the last place is 1, so
                    // the bits 0x4B400000 + sv read as the float 1.5*2^23 + sv
                    // for |sv| < 2^22 (|sv| <= c <= 512 here); subtracting
                    // 1.5 * 2^23 is then exact.
                    const float fs = __int_as_float(0x4B400000 + sv) - 12582912.0f;
                    op[p][co_off] = fmaf(g, fs, bb);
                }
            }
        }
        u = (int64_t)(pb + 1) * cout;
    }
}

}  // namespace bnn
