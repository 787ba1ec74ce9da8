// Binary weights x real activations GEMV: "Extreme Quantization: Binary,
// Ternary & 1-bit LLMs", Binary Neural Networks, eq. (1)-(2):
//   y[n] = alpha[n] * sum_k sign(w_nk) * x_k,
// each term +x_k or -x_k (no multiplication), with the packed weights of
// bnn_pack_sign (bit 1 = -1, pad bits 0) and a real x.
//
// Add table.  For every group of 4 consecutive x values (one nibble of a
// packed word) the 16 signed sums +-x0 +-x1 +-x2 +-x3 are built once per CTA
// in shared memory (entry m negates element j iff bit j of m is set; pad
// elements are 0).  A row's sum is then one table lookup and one add per 4
// weights.
//
// Work split.  One CTA per SM walks groups of 32 rows, and the table is
// built once per CTA.  Warp w takes the 16-byte chunks w, w + 16, w + 32, ...
// of each row (K split 16 ways) and lane l is row l of the group, so the 32
// lanes of a warp always look up the same table row (16 consecutive floats):
// no bank conflicts.  The first weight batch is loaded before the table is
// built, and the next group's batch while the current one is summed.  The 16
// partial sums of a row meet in shared memory.  A CTA holds 66 KB of shared
// memory at K = 4096, so two consecutive launches fit on one SM.
//
// Launched with programmatic dependent launch, like the XNOR GEMV: with static
// weights the W loads precede the wait for the previous grid, with static
// inputs the table and the product do too, and with all three flags only the
// exit waits.
#pragma once

#include "common.cuh"

namespace bnn {
namespace bwg {
constexpr int WARPS = 16;                 // K slices
constexpr int THREADS = WARPS * 32;
constexpr int NB = 2;                     // chunks per lane per batch (loads in flight)
constexpr int MAX_KW = 384;               // table of MAX_KW * 8 groups x 64 B = 192 KiB
__host__ __device__ constexpr int smem_bytes(int kw) { return 64 + kw * 8 * 64 + WARPS * 32 * 4; }
}  // namespace bwg

template <typename XT>
__global__ void __launch_bounds__(bwg::THREADS)
bw_gemv_kernel(const uint32_t* __restrict__ W, int64_t ldw, const XT* __restrict__ x, int N, int K, int kw,
               const float* __restrict__ alpha, float* __restrict__ y, int prefetch, int xstatic, int dependent) {
    using namespace bwg;
    extern __shared__ __align__(16) float bw_smem[];
    // [kw * 8][16] with 64-byte aligned rows: the entry of group g, nibble n is
    // at byte offset (g * 64) | (n * 4).
    float* table = bw_smem + (((64u - (smem_u32(bw_smem) & 63u)) & 63u) >> 2);
    const char* tbytes = reinterpret_cast<const char*>(table);
    float* part = table + kw * 8 * 16;                        // [WARPS][32]
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int nch = kw / 4;                                   // 16-byte chunks per row
    const int groups = (N + 31) / 32;                         // row groups of 32
    grid_dependents_launch();

    // A CTA walks the row groups blockIdx.x, + gridDim.x, ...; the table is
    // built once per CTA and the first weight batch of the next row group is
    // loaded while the current one is summed.
    uint4 v[NB], vn[NB];
    auto load_batch = [&](uint4 (&dst)[NB], int rgi, int cb) {
        const int row = rgi * 32 + lane;
        #pragma unroll
        for (int i = 0; i < NB; ++i) {
            const int c = cb + WARPS * i;
            dst[i] = (rgi < groups && row < N && c < nch) ? ldg_stream_v4(W + (int64_t)row * ldw + 4 * c)
                                                          : make_uint4(0u, 0u, 0u, 0u);
        }
    };
    auto build_table = [&]() {
        for (int g = threadIdx.x; g < kw * 8; g += THREADS) {
            float e[4];
            #pragma unroll
            for (int j = 0; j < 4; ++j) {
                const int k = 4 * g + j;
                e[j] = k < K ? to_float(x[k]) : 0.0f;
            }
            float p01[4], p23[4];
            #pragma unroll
            for (int b = 0; b < 4; ++b) {
                p01[b] = ((b & 1) ? -e[0] : e[0]) + ((b & 2) ? -e[1] : e[1]);
                p23[b] = ((b & 1) ? -e[2] : e[2]) + ((b & 2) ? -e[3] : e[3]);
            }
            float4* t = reinterpret_cast<float4*>(table + g * 16);
            #pragma unroll
            for (int h = 0; h < 4; ++h)      // entries 4h .. 4h+3: p23 index h, p01 index 0..3
                t[h] = make_float4(p01[0] + p23[h], p01[1] + p23[h], p01[2] + p23[h], p01[3] + p23[h]);
        }
    };
    const bool late_wait = prefetch && xstatic;
    if (prefetch) load_batch(v, blockIdx.x, warp);
    if (xstatic) build_table();
    if (dependent == 1 && !late_wait) grid_dependency_wait();
    if (!prefetch) load_batch(v, blockIdx.x, warp);
    if (!xstatic) build_table();
    __syncthreads();

    bool first = true;
    for (int rgi = blockIdx.x; rgi < groups; rgi += gridDim.x) {
        load_batch(vn, rgi + gridDim.x, warp);                // next row group, first batch
        float acc[4] = {0.f, 0.f, 0.f, 0.f};
        for (int cb = warp; cb < nch; cb += WARPS * NB) {
            if (cb != warp) load_batch(v, rgi, cb);           // later batches (K > 4096)
            #pragma unroll
            for (int i = 0; i < NB; ++i) {
                const int c = cb + WARPS * i;
                if (c >= nch) break;
                const uint32_t wq[4] = {v[i].x, v[i].y, v[i].z, v[i].w};
                #pragma unroll
                for (int q = 0; q < 4; ++q) {
                    const uint32_t grow = (uint32_t)((4 * c + q) * 8) * 64u;   // byte offset of the word's groups
                    #pragma unroll
                    for (int j = 0; j < 8; ++j) {
                        // nibble j moved to bits 2..5 (byte offset nibble * 4)
                        const uint32_t nib4 = j == 0 ? (wq[q] << 2) : (wq[q] >> (4 * j - 2));
                        acc[j & 3] += *reinterpret_cast<const float*>(tbytes + ((grow + 64u * j) | (nib4 & 0x3Cu)));
                    }
                }
            }
        }
        part[warp * 32 + lane] = (acc[0] + acc[1]) + (acc[2] + acc[3]);
        __syncthreads();
        if (threadIdx.x < 32) {
            const int row = rgi * 32 + lane;
            float s = 0.0f;
            #pragma unroll
            for (int w = 0; w < WARPS; ++w) s += part[w * 32 + lane];
            if (first && dependent == 1 && late_wait) grid_dependency_wait();
            if (row < N) y[row] = alpha[row] * s;
        }
        __syncthreads();                                      // part[] is rewritten next round
        first = false;
        #pragma unroll
        for (int i = 0; i < NB; ++i) v[i] = vn[i];
    }
    if (dependent == 2) grid_dependency_wait();
}

}  // namespace bnn
