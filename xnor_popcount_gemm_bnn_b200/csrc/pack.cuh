// Sign-and-pack kernels: real tensors -> packed sign bits (+ per-row alpha).
//
// sign(): "Extreme Quantization: Binary, Ternary & 1-bit LLMs", Notation and
// XNOR-Net eq. (4).  Encoding and packing: "First Principles: Why Binary Ops
// Can Be Exponentially Faster", section 1 (bit 0 = +1, bit 1 = -1, pad = +1).
// alpha = (1/K) sum_k |w_k|: "Extreme Quantization ...", eq. (1).
//
// All three kernels are bound by reading the real input from HBM (4 bytes
// in, 1/8 byte out per fp32 element); they use 16-byte vector loads,
// coalesced across the warp, with several loads in flight per lane.
#pragma once

#include "common.cuh"

namespace bnn {

// One warp per row.  A lane loads E = 16/sizeof(T) consecutive elements per
// 16-byte vector; a warp-wide load covers 32*E elements = E words.  Lane l's
// E sign bits land at bit E*(l % G) of word l / G (G = 32/E lanes per word);
// an OR-butterfly over those G lanes assembles the word.
template <typename T, int U>
__global__ void __launch_bounds__(256)
pack_sign_rows_kernel(const T* __restrict__ x, int64_t rows, int64_t K, int64_t ld_x,
                      uint32_t* __restrict__ packed, int64_t ldp, float* __restrict__ alpha_out,
                      int64_t kw, bool vec_ok) {
    constexpr int E = 16 / (int)sizeof(T);
    constexpr int G = 32 / E;
    constexpr int CH = 32 * E;  // elements per warp chunk
    const int lane = threadIdx.x & 31;
    const int64_t row = (int64_t)blockIdx.x * (blockDim.x >> 5) + (threadIdx.x >> 5);
    if (row >= rows) return;
    const T* xr = x + row * ld_x;
    uint32_t* pr = packed + row * ldp;
    const int64_t nchunks = (kw * 32 + CH - 1) / CH;
    double asum = 0.0;

    for (int64_t c0 = 0; c0 < nchunks; c0 += U) {
        float v[U][E];
        #pragma unroll
        for (int u = 0; u < U; ++u) {
            const int64_t base = (c0 + u) * CH + (int64_t)lane * E;
            if (vec_ok && base + E <= K) {
                uint4 q = ldg_stream_v4(xr + base);
                const T* e = reinterpret_cast<const T*>(&q);
                #pragma unroll
                for (int i = 0; i < E; ++i) v[u][i] = to_float(e[i]);
            } else {
                #pragma unroll
                for (int i = 0; i < E; ++i)
                    v[u][i] = (base + i < K) ? to_float(xr[base + i]) : 0.0f;
            }
        }
        #pragma unroll
        for (int u = 0; u < U; ++u) {
            const int64_t chunk = c0 + u;
            if (chunk >= nchunks) break;
            uint32_t bits = 0;
            #pragma unroll
            for (int i = 0; i < E; ++i) {
                bits |= neg_bit(v[u][i]) << i;
                asum += fabs((double)v[u][i]);  // elements past K were loaded as 0
            }
            bits <<= E * (lane % G);
            #pragma unroll
            for (int off = 1; off < G; off <<= 1) bits |= __shfl_xor_sync(0xffffffffu, bits, off);
            const int64_t wi = chunk * E + lane / G;
            if ((lane % G) == 0 && wi < kw) pr[wi] = bits;
        }
    }
    if (alpha_out != nullptr) {
        #pragma unroll
        for (int off = 16; off >= 1; off >>= 1) asum += __shfl_xor_sync(0xffffffffu, asum, off);
        if (lane == 0) alpha_out[row] = (float)(asum / (double)K);
    }
}

// NCHW real activations -> per-pixel channel words [n, h, w, cw].
// One thread builds the word j of 8 consecutive pixels: 32 channel loads of 8
// pixels each (one 16-byte bf16 vector or two fp32 vectors), bit q of the
// pixel's word = sign bit of channel 32*j + q.  Threads are ordered (pixel
// group, word) so that a warp writes a contiguous stretch of the output.
template <typename T>
__global__ void __launch_bounds__(256)
pack_sign_nchw_kernel(const T* __restrict__ x, int64_t n, int64_t c, int64_t hw, int64_t cw,
                      uint32_t* __restrict__ out, bool vec_ok) {
    constexpr int P = 8;
    const int64_t groups = (hw + P - 1) / P;
    const int64_t tid = (int64_t)blockIdx.x * blockDim.x + threadIdx.x;
    if (tid >= n * groups * cw) return;
    const int64_t j = tid % cw;
    const int64_t g = (tid / cw) % groups;
    const int64_t b = tid / (cw * groups);
    const int64_t p0 = g * P;
    const int np = (int)(hw - p0 < P ? hw - p0 : P);
    uint32_t bits[P];
    #pragma unroll
    for (int p = 0; p < P; ++p) bits[p] = 0;
    const int qmax = (int)(c - 32 * j < 32 ? c - 32 * j : 32);
    #pragma unroll 8
    for (int q = 0; q < qmax; ++q) {
        const T* src = x + ((b * c + 32 * j + q) * hw + p0);
        float v[P];
        if (vec_ok && np == P) {
            if constexpr (sizeof(T) == 2) {
                uint4 r = ldg_stream_v4(src);
                const T* e = reinterpret_cast<const T*>(&r);
                #pragma unroll
                for (int p = 0; p < P; ++p) v[p] = to_float(e[p]);
            } else {
                uint4 r0 = ldg_stream_v4(src), r1 = ldg_stream_v4(src + 4);
                const T* e0 = reinterpret_cast<const T*>(&r0);
                const T* e1 = reinterpret_cast<const T*>(&r1);
                #pragma unroll
                for (int p = 0; p < 4; ++p) { v[p] = to_float(e0[p]); v[p + 4] = to_float(e1[p]); }
            }
        } else {
            #pragma unroll
            for (int p = 0; p < P; ++p) v[p] = (p < np) ? to_float(src[p]) : 0.0f;
        }
        #pragma unroll
        for (int p = 0; p < P; ++p) bits[p] |= neg_bit(v[p]) << q;
    }
    uint32_t* dst = out + ((b * hw + p0) * cw + j);
    #pragma unroll
    for (int p = 0; p < P; ++p)
        if (p < np) dst[(int64_t)p * cw] = bits[p];
}

// OIHW 3x3 filters -> packed rows in (kh, kw, c) order, one warp per output
// channel; lane = channel within a 32-channel word.  alpha over the 9*cin
// true weights (eq. (1): one scale per filter).
template <typename T>
__global__ void __launch_bounds__(256)
pack_conv3x3_weights_kernel(const T* __restrict__ w, int64_t cout, int64_t cin,
                            uint32_t* __restrict__ packed, int64_t ldp, float* __restrict__ alpha_out) {
    const int lane = threadIdx.x & 31;
    const int64_t co = (int64_t)blockIdx.x * (blockDim.x >> 5) + (threadIdx.x >> 5);
    if (co >= cout) return;
    const int64_t cw = (cin + 31) / 32;
    const int64_t words = 9 * cw;
    const int64_t ldk = (words + 3) / 4 * 4;
    uint32_t* pr = packed + co * ldp;
    double asum = 0.0;
    for (int t = 0; t < 9; ++t) {
        for (int64_t j = 0; j < cw; ++j) {
            const int64_t ch = 32 * j + lane;
            const float v = (ch < cin) ? to_float(w[(co * cin + ch) * 9 + t]) : 0.0f;
            asum += fabs((double)v);
            const uint32_t word = __ballot_sync(0xffffffffu, v < 0.0f);
            if (lane == 0) pr[t * cw + j] = word;
        }
    }
    for (int64_t wi = words + lane; wi < ldk; wi += 32) pr[wi] = 0u;
    if (alpha_out != nullptr) {
        #pragma unroll
        for (int off = 16; off >= 1; off >>= 1) asum += __shfl_xor_sync(0xffffffffu, asum, off);
        if (lane == 0) alpha_out[co] = (float)(asum / (double)(9 * cin));
    }
}

}  // namespace bnn
