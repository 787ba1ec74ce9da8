// Binary weights x INT8 activations GEMV ("Extreme Quantization: Binary,
// Ternary & 1-bit LLMs": Binary Neural Networks, eq. (1)-(2) -- each term is
// +x_k or -x_k; the BitNet section -- activations quantised to INT8; eq. (8)
// -- one scale for the whole weight matrix):
//   acc[n]   = sum_k sign(W[n,k]) * x_k          (exact, int32)
//   y_f32[n] = fp32( fp32(alpha_n * x_scale) * fp32(acc[n]) )
// with alpha per output row (eq. (1)) or one alpha for the matrix (eq. (8)).
//
// With b_k the packed bit (1 = -1), sign(w_k) x_k = x_k - 2 b_k x_k, so
// acc = sum x - 2 sum_{b=1} x.  A sign-replicating PRMT of the packed word
// shifted left by s gives bytes 0xFF (-1) / 0x00 for the four elements
// 7-s, 15-s, 23-s, 31-s (the order the tensor-core unpack uses); one signed
// dp4a against the same four x bytes adds -sum_{b=1} x over them.  So per 4
// weights: a shift, a PRMT and a dp4a.  x is staged once per CTA in shared
// memory already permuted into that byte order (8 words per packed word),
// and each lane keeps the 32 words of its 128-element chunk in registers,
// with their plain sum from 32 more dp4a against 0x01010101.
//
// Work split as the XNOR GEMV: lane l takes the 16-byte chunks l, l + LPR, ...
// of a row (a warp-wide load is one contiguous row segment), U rows per warp
// with all loads in flight, row sums by redux / shuffles.  The dependency
// flags of bnn_xnor_gemv_ex apply.
#pragma once

#include "common.cuh"

namespace bnn {
namespace bwi8 {
constexpr int THREADS = 256;
constexpr int WARPS = THREADS / 32;
constexpr int U = 8;                       // row groups per warp, all loads in flight
constexpr int MAX_KW = 1536;               // K <= 49152: permuted x in 48 KiB of shared memory
}  // namespace bwi8

template <int U>
__global__ void __launch_bounds__(bwi8::THREADS)
bw_gemv_i8_kernel(const uint32_t* __restrict__ W, int64_t ldw, const int8_t* __restrict__ x, int N, int K, int kw,
                  const float* __restrict__ alpha, int alpha_per_row, const float* __restrict__ x_scale,
                  int32_t* __restrict__ y_i32, float* __restrict__ y_f32, int prefetch, int xstatic,
                  int dependent) {
    using namespace bwi8;
    extern __shared__ __align__(16) uint32_t xp[];             // [kw][8]: permuted x, 4 bytes per word
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int nch = kw / 4;
    int lpr = 1;
    while (lpr < 32 && lpr < nch) lpr <<= 1;
    const int rpi = 32 / lpr;
    const int li = lane & (lpr - 1), sub = lane / lpr;
    const int np = (nch + lpr - 1) / lpr;                      // chunks per lane
    const int rows_per_batch = U * rpi;
    const int total_warps = (int)gridDim.x * WARPS;
    const int gw = (int)blockIdx.x * WARPS + warp;
    grid_dependents_launch();

    uint4 v[U];
    float al[U];                                               // alpha of the rows this lane stores (li == 0)
    // The first pass also reads the rows' alpha (the weights and their scale
    // are read together).
    auto load_pass = [&](int row0, int p) {
        const int c = li + lpr * p;
        #pragma unroll
        for (int u = 0; u < U; ++u) {
            const int r = row0 + u * rpi;
            v[u] = (r < N && c < nch) ? ldg_stream_v4(W + (int64_t)r * ldw + 4 * c) : make_uint4(0u, 0u, 0u, 0u);
            if (p == 0) al[u] = (li == 0 && y_f32 != nullptr && r < N) ? alpha[alpha_per_row ? r : 0] : 0.0f;
        }
    };
    // Word w of x (elements 32 w .. 32 w + 31, zero past K) -> 8 permuted
    // words: word s holds the bytes of elements 7-s, 15-s, 23-s, 31-s.
    auto stage_x = [&]() {
        for (int w = threadIdx.x; w < kw; w += THREADS) {
            uint32_t b[8];
            const int k0 = 32 * w;
            if (k0 + 32 <= K && (reinterpret_cast<uintptr_t>(x + k0) & 15) == 0) {
                const uint4 lo = *reinterpret_cast<const uint4*>(x + k0);
                const uint4 hi = *reinterpret_cast<const uint4*>(x + k0 + 16);
                b[0] = lo.x; b[1] = lo.y; b[2] = lo.z; b[3] = lo.w;
                b[4] = hi.x; b[5] = hi.y; b[6] = hi.z; b[7] = hi.w;
            } else {
                #pragma unroll
                for (int i = 0; i < 8; ++i) {
                    uint32_t q = 0;
                    #pragma unroll
                    for (int j = 0; j < 4; ++j) {
                        const int k = k0 + 4 * i + j;
                        if (k < K) q |= (uint32_t)(uint8_t)x[k] << (8 * j);
                    }
                    b[i] = q;
                }
            }
            // element e is byte e % 4 of b[e / 4]
            #pragma unroll
            for (int s = 0; s < 8; ++s) {
                uint32_t q = 0;
                #pragma unroll
                for (int j = 0; j < 4; ++j) {
                    const int e = 8 * j + 7 - s;
                    q |= ((b[e >> 2] >> (8 * (e & 3))) & 0xFFu) << (8 * j);
                }
                xp[w * 8 + s] = q;
            }
        }
    };

    const bool late_wait = prefetch && xstatic;
    int row0 = gw * rows_per_batch + sub;
    if (prefetch) load_pass(row0, 0);
    if (xstatic) stage_x();
    if (dependent == 1 && !late_wait) grid_dependency_wait();
    if (!prefetch) load_pass(row0, 0);
    if (!xstatic) stage_x();
    __syncthreads();

    bool first = true;
    for (int b0 = gw * rows_per_batch; b0 < N; b0 += total_warps * rows_per_batch) {
        row0 = b0 + sub;
        int acc[U];
        #pragma unroll
        for (int u = 0; u < U; ++u) acc[u] = 0;
        int xsum = 0;
        for (int p = 0; p < np; ++p) {
            if (!first || p > 0) load_pass(row0, p);
            const int c = li + lpr * p;
            uint32_t xr[32];
            if (c < nch) {
                const uint4* src = reinterpret_cast<const uint4*>(xp + 32 * c);
                #pragma unroll
                for (int i = 0; i < 8; ++i) {
                    const uint4 q = src[i];
                    xr[4 * i] = q.x; xr[4 * i + 1] = q.y; xr[4 * i + 2] = q.z; xr[4 * i + 3] = q.w;
                }
            } else {
                #pragma unroll
                for (int i = 0; i < 32; ++i) xr[i] = 0u;
            }
            #pragma unroll
            for (int i = 0; i < 32; ++i) xsum = __dp4a((int)xr[i], 0x01010101, xsum);
            #pragma unroll
            for (int u = 0; u < U; ++u) {
                const uint32_t wq[4] = {v[u].x, v[u].y, v[u].z, v[u].w};
                #pragma unroll
                for (int q = 0; q < 4; ++q) {
                    #pragma unroll
                    for (int s = 0; s < 8; ++s) {
                        uint32_t m;
                        asm("prmt.b32 %0, %1, 0, 0xBA98;" : "=r"(m) : "r"(wq[q] << s));
                        acc[u] = __dp4a((int)m, (int)xr[8 * q + s], acc[u]);
                    }
                }
            }
        }
        #pragma unroll
        for (int u = 0; u < U; ++u) {
            int t = xsum + 2 * acc[u];                         // sum x - 2 sum_{b=1} x, this lane's chunks
            if (lpr == 32) {
                t = __reduce_add_sync(0xffffffffu, t);
            } else {
                for (int off = lpr >> 1; off >= 1; off >>= 1) t += __shfl_xor_sync(0xffffffffu, t, off);
            }
            acc[u] = t;
        }
        if (first && dependent == 1 && late_wait) grid_dependency_wait();
        first = false;
        if (li == 0) {
            const float xs = x_scale != nullptr ? *x_scale : 1.0f;
            #pragma unroll
            for (int u = 0; u < U; ++u) {
                const int r = row0 + u * rpi;
                if (r < N) {
                    if (y_i32 != nullptr) y_i32[r] = acc[u];
                    if (y_f32 != nullptr) y_f32[r] = (al[u] * xs) * (float)acc[u];
                }
            }
        }
    }
    if (dependent == 2) exit_after_previous_grid();
}

}  // namespace bnn
