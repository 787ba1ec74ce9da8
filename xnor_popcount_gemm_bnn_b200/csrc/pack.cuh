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
// A pair of threads builds word j of 8 consecutive pixels: each takes 16 of
// the word's 32 channels (16-byte loads of 8 pixels, all issued before any is
// used), and one shuffle merges the halves.  Bit q of a pixel's word is the
// sign bit of channel 32*j + q.  Threads are ordered (pixel group, word,
// half), so a warp reads 4 channel planes x 128 contiguous bytes per load and
// writes a contiguous stretch of the output.
template <typename T>
__global__ void __launch_bounds__(128)
pack_sign_nchw_kernel(const T* __restrict__ x, int64_t n, int64_t c, int64_t hw, int64_t cw,
                      uint32_t* __restrict__ out, bool vec_ok) {
    constexpr int P = 8, CH = 16;
    const int64_t groups = (hw + P - 1) / P;
    const int64_t total = n * groups * cw * 2;               // even: partners live or die together
    const int64_t tid = (int64_t)blockIdx.x * blockDim.x + threadIdx.x;
    const bool live = tid < total;
    const int half = (int)(tid & 1);
    const int64_t u = (live ? tid : 0) >> 1;
    const int64_t j = u % cw;
    const int64_t g = (u / cw) % groups;
    const int64_t b = u / (cw * groups);
    const int64_t p0 = g * P;
    const int np = (int)(hw - p0 < P ? hw - p0 : P);
    const int64_t c0 = 32 * j + CH * half;
    const int nq = (int)(c - c0 <= 0 ? 0 : (c - c0 < CH ? c - c0 : CH));
    const T* src = x + ((b * c + c0) * hw + p0);
    uint32_t bits[P];
    #pragma unroll
    for (int p = 0; p < P; ++p) bits[p] = 0;
    if (vec_ok) {                                            // hw % 8 == 0: np == P
        constexpr int VPC = sizeof(T) == 2 ? 1 : 2;         // 16-byte vectors per channel
        constexpr int QR = 16 / VPC;                         // channels per round of 16 loads
        #pragma unroll
        for (int q0 = 0; q0 < CH; q0 += QR) {
            // Plain read-only loads (not volatile asm), so the scheduler keeps
            // all 16 in flight before the first is used.
            uint4 r[16];
            #pragma unroll
            for (int i = 0; i < 16; ++i) {
                const int q = q0 + i / VPC;
                const uint4* a = reinterpret_cast<const uint4*>(src + q * hw + (i % VPC) * (8 / VPC));
                r[i] = (nq == CH || q < nq) ? __ldg(a) : make_uint4(0u, 0u, 0u, 0u);
            }
            #pragma unroll
            for (int i = 0; i < 16; ++i) {
                const T* e = reinterpret_cast<const T*>(&r[i]);
                #pragma unroll
                for (int k = 0; k < 8 / VPC; ++k)
                    bits[(i % VPC) * (8 / VPC) + k] |= neg_bit(to_float(e[k])) << (q0 + i / VPC);
            }
        }
    } else {
        for (int q = 0; q < nq; ++q) {
            #pragma unroll
            for (int p = 0; p < P; ++p)
                if (p < np) bits[p] |= neg_bit(to_float(src[q * hw + p])) << q;
        }
    }
    #pragma unroll
    for (int p = 0; p < P; ++p) {
        bits[p] <<= CH * half;
        bits[p] |= __shfl_xor_sync(0xffffffffu, bits[p], 1);
    }
    if (!live) return;
    uint32_t* dst = out + ((b * hw + p0) * cw + j);
    #pragma unroll
    for (int p = 0; p < P; ++p)
        if ((p >> 2) == half && p < np) dst[(int64_t)p * cw] = bits[p];
}

// NCHW real activations -> per-pixel channel words [n, h, w, cw], staged by
// TMA.  The input is viewed as a 2-D tensor [n*c rows, hw columns]; a chunk is
// PX consecutive pixels of one image with all its channels, loaded as
// nbox boxes of [cb channel rows x PX pixels] into one of STAGES shared-memory
// buffers.  Every CTA keeps STAGES - 1 chunks in flight while it converts
// the current one, so the copies, not the threads' registers, carry the
// memory-level parallelism.  A thread converts 2 adjacent pixels per channel
// (one 2-pixel shared load); columns past hw arrive zero-filled and are not
// stored; rows past the image's c channels are ignored.
namespace pk {
constexpr int THREADS = 128;
constexpr int STAGES = 3;
}  // namespace pk

template <typename T>
__global__ void __launch_bounds__(pk::THREADS)
pack_sign_nchw_tma_kernel(const __grid_constant__ CUtensorMap tmx, int n, int c, int hw, int cw, int px, int cb,
                          int nbox, uint32_t* __restrict__ out) {
    extern __shared__ uint8_t smem_raw[];
    uint8_t* smem = smem_raw + ((128u - (smem_u32(smem_raw) & 127u)) & 127u);
    const int stage_bytes = nbox * cb * px * (int)sizeof(T);
    __shared__ uint64_t full[pk::STAGES];
    const int chunks_per_img = (hw + px - 1) / px;
    const int chunks = n * chunks_per_img;
    const int mine = chunks > (int)blockIdx.x ? (chunks - 1 - (int)blockIdx.x) / (int)gridDim.x + 1 : 0;
    if (threadIdx.x == 0) {
        for (int s = 0; s < pk::STAGES; ++s) mbar_init(&full[s], 1);
        fence_mbarrier_init();
        prefetch_tensormap(&tmx);
    }
    __syncthreads();
    auto issue = [&](int i) {               // chunk i of this CTA into stage i % STAGES
        const int ch = (int)blockIdx.x + i * (int)gridDim.x;
        const int b = ch / chunks_per_img, p0 = (ch - b * chunks_per_img) * px;
        uint64_t* bar = &full[i % pk::STAGES];
        uint8_t* dst = smem + (i % pk::STAGES) * stage_bytes;
        mbar_arrive_expect_tx(bar, (uint32_t)stage_bytes);
        for (int k = 0; k < nbox; ++k)
            tma_load_2d(dst + k * cb * px * (int)sizeof(T), &tmx, p0, b * c + k * cb, bar);
    };
    if (threadIdx.x == 0)
        for (int i = 0; i < pk::STAGES - 1 && i < mine; ++i) issue(i);
    int issued = mine < pk::STAGES - 1 ? mine : pk::STAGES - 1;
    int i = 0;
    for (; i < mine; ++i) {
        if (threadIdx.x == 0 && issued < mine) { issue(issued); ++issued; }
        const bool ok = mbar_wait_bounded(&full[i % pk::STAGES], (uint32_t)((i / pk::STAGES) & 1));
        if (__syncthreads_or(!ok)) break;
        const int ch = (int)blockIdx.x + i * (int)gridDim.x;
        const int b = ch / chunks_per_img, p0 = (ch - b * chunks_per_img) * px;
        const T* st = reinterpret_cast<const T*>(smem + (i % pk::STAGES) * stage_bytes);
        for (int pp = threadIdx.x; pp < px / 2; pp += pk::THREADS) {
            const int p = p0 + 2 * pp;
            if (p >= hw) break;
            uint32_t* dst = out + ((int64_t)b * hw + p) * cw;
            for (int j = 0; j < cw; ++j) {
                uint32_t w0 = 0, w1 = 0;
                const int qn = c - 32 * j < 32 ? c - 32 * j : 32;
                #pragma unroll 8
                for (int q = 0; q < qn; ++q) {
                    const T* e = st + (32 * j + q) * px + 2 * pp;
                    w0 |= neg_bit(to_float(e[0])) << q;
                    w1 |= neg_bit(to_float(e[1])) << q;
                }
                dst[j] = w0;
                if (p + 1 < hw) dst[cw + j] = w1;
            }
        }
        __syncthreads();                     // stage i % STAGES may be refilled
    }
    // After a time-out, let the copies still in flight land before exiting.
    if (threadIdx.x == 0)
        for (int k = i + 1; k < issued; ++k)
            mbar_wait_bounded(&full[k % pk::STAGES], (uint32_t)((k / pk::STAGES) & 1));
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
