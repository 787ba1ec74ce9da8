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
// One warp task = word j of 32 consecutive pixels of one image.  Lane q reads
// channel 32*j + q over those pixels (64 contiguous bytes of bf16, 128 of
// fp32, as 16-byte vectors all in flight together), and one __ballot_sync
// per pixel collects the word: bit q = sign of channel 32*j + q, which is
// exactly the packed layout (LSB = lowest channel).  Lane p keeps the word
// of pixel p and stores it.  Tasks are ordered (image, pixel group, word),
// so consecutive warps stream consecutive stretches of the same channel rows.
template <typename T>
__global__ void __launch_bounds__(256)
pack_sign_nchw_kernel(const T* __restrict__ x, int64_t n, int64_t c, int64_t hw, int64_t cw,
                      uint32_t* __restrict__ out, bool vec_ok) {
    constexpr int PX = 32;                        // pixels per task
    constexpr int E = 16 / (int)sizeof(T);        // elements per 16-byte vector
    constexpr int NV = PX / E;                    // vectors per lane
    const int lane = threadIdx.x & 31;
    const int64_t groups = (hw + PX - 1) / PX;
    const int64_t task = ((int64_t)blockIdx.x * blockDim.x + threadIdx.x) >> 5;
    if (task >= n * groups * cw) return;          // whole warps leave together
    const int64_t j = task % cw;
    const int64_t g = (task / cw) % groups;
    const int64_t b = task / (cw * groups);
    const int64_t p0 = g * PX;
    const int np = (int)(hw - p0 < PX ? hw - p0 : PX);
    const int64_t ch = 32 * j + lane;
    const bool live = ch < c;
    const T* src = x + ((b * c + (live ? ch : 0)) * hw + p0);
    uint4 v[NV];
    if (vec_ok && np == PX) {
        #pragma unroll
        for (int i = 0; i < NV; ++i)
            v[i] = live ? __ldg(reinterpret_cast<const uint4*>(src + i * E)) : make_uint4(0u, 0u, 0u, 0u);
    } else {
        #pragma unroll
        for (int i = 0; i < NV; ++i) {
            union { uint4 u; T e[E]; } t;
            #pragma unroll
            for (int k = 0; k < E; ++k) t.e[k] = (live && i * E + k < np) ? src[i * E + k] : T(0.0f);
            v[i] = t.u;
        }
    }
    uint32_t mine = 0;
    #pragma unroll
    for (int i = 0; i < NV; ++i) {
        const T* e = reinterpret_cast<const T*>(&v[i]);
        #pragma unroll
        for (int k = 0; k < E; ++k) {
            const uint32_t word = __ballot_sync(0xffffffffu, to_float(e[k]) < 0.0f);
            if (lane == i * E + k) mine = word;
        }
    }
    if (lane < np) out[(b * hw + p0 + lane) * cw + j] = mine;
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
