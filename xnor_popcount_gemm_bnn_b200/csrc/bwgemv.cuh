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
// Work split.  A warp reads whole rows: lane l takes the 16-byte chunks
// l, l + 32, ... of a row (LPR lanes per row when a row has fewer than 32
// chunks), so one warp-wide load is one contiguous 512-byte row segment.
// The table is laid out [pass][group][entry][lane]: the entries a lane can
// ever look up (the groups of its own chunks) sit in bank `lane`, so the 32
// lookups of a warp never conflict, whatever the nibbles.  Each warp issues
// the loads of U rows before the table is built (the weight stream overlaps
// it), sums each row on 4 accumulators per lane, and adds the lanes of a
// row with a butterfly of shuffles -- no block barrier after the table.
//
// Launched with programmatic dependent launch, like the XNOR GEMV: with static
// weights the first W loads precede the wait for the previous grid, with
// static inputs the table and the product do too (only the store waits), and
// with all three flags only the exit waits.
#pragma once

#include "common.cuh"

namespace bnn {
namespace bwg {
constexpr int WARPS = 16;
constexpr int THREADS = WARPS * 32;
constexpr int U = 5;                      // row groups per warp per batch, all loads in flight
constexpr int MAX_KW = 384;               // 3 passes of 128 words: 192 KiB of table
// Passes: how many chunks each lane takes per row (rows of up to 128 words
// take one).  The table holds 32 groups x 16 entries x 32 lanes per pass.
__host__ __device__ constexpr int passes(int kw) { return (kw + 127) / 128; }
constexpr int PASS_FLOATS = 32 * 16 * 32;
// The slice of x one pass reads (32 chunks x 128 elements), staged as fp32
// with one pad float after every 128 elements, so that lanes reading 128
// elements apart fall on distinct banks.
constexpr int XS_FLOATS = 4096 + 32;
__host__ __device__ constexpr int smem_bytes(int kw) { return (passes(kw) * PASS_FLOATS + XS_FLOATS) * 4 + 128; }
}  // namespace bwg

template <typename XT>
__global__ void __launch_bounds__(bwg::THREADS, 2)
bw_gemv_kernel(const uint32_t* __restrict__ W, int64_t ldw, const XT* __restrict__ x, int N, int K, int kw,
               const float* __restrict__ alpha, float* __restrict__ y, int prefetch, int xstatic, int dependent) {
    using namespace bwg;
    extern __shared__ __align__(16) float bw_smem[];
    float* table = bw_smem + (((128u - (smem_u32(bw_smem) & 127u)) & 127u) >> 2);
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int nch = kw / 4;                                   // 16-byte chunks per row
    int lpr = 1;                                              // lanes per row: a power of two >= min(nch, 32)
    while (lpr < 32 && lpr < nch) lpr <<= 1;
    const int rpi = 32 / lpr;                                 // rows per warp-wide load
    const int li = lane & (lpr - 1), sub = lane / lpr;
    const int np = passes(kw);
    float* xs = table + np * PASS_FLOATS;                     // x as fp32, padded
    const int rows_per_batch = U * rpi;                       // rows of one warp per batch
    const int64_t total_warps = (int64_t)gridDim.x * WARPS;
    const int64_t gw = (int64_t)blockIdx.x * WARPS + warp;
    grid_dependents_launch();

    uint4 v[U];
    auto row_of = [&](int64_t batch, int u) -> int64_t {
        return ((gw + batch * total_warps) * U + u) * rpi + sub;
    };
    auto load_pass = [&](int64_t batch, int p) {
        const int c = li + lpr * p;
        #pragma unroll
        for (int u = 0; u < U; ++u) {
            const int64_t r = row_of(batch, u);
            v[u] = (r < N && c < nch) ? ldg_stream_v4(W + r * ldw + 4 * c) : make_uint4(0u, 0u, 0u, 0u);
        }
    };
    // Per pass: the pass's slice of x -> shared fp32 (coalesced 16-byte loads
    // when x is aligned), then that pass's table: entry (p, t, m, l) =
    // sum_j (bit j of m ? -x : +x)[k0 + j], k0 = 128 c + 4 t with
    // c = (l mod lpr) + lpr p the chunk lane l reads in pass p.  A pass reads
    // the 4096 elements starting at 4096 p (several passes happen only with
    // lpr = 32).  Thread (slot, l) builds groups t = slot, slot + 16; a warp
    // writes 32 consecutive floats per entry.
    auto build_table = [&]() {
        constexpr int E = 16 / (int)sizeof(XT);
        const int kpad = kw * 32;
        const bool vec = (reinterpret_cast<uintptr_t>(x) & 15) == 0;
        for (int p = 0; p < np; ++p) {
            const int kb = 4096 * p;
            if (p > 0) __syncthreads();                       // the previous pass is done reading xs
            for (int i0 = E * (int)threadIdx.x; i0 < 4096 && kb + i0 < kpad; i0 += E * THREADS) {
                const int k = kb + i0;
                float e[E];
                if (vec && k + E <= K) {
                    const uint4 q = *reinterpret_cast<const uint4*>(x + k);
                    const XT* el = reinterpret_cast<const XT*>(&q);
                    #pragma unroll
                    for (int i = 0; i < E; ++i) e[i] = to_float(el[i]);
                } else {
                    #pragma unroll
                    for (int i = 0; i < E; ++i) e[i] = k + i < K ? to_float(x[k + i]) : 0.0f;
                }
                #pragma unroll
                for (int i = 0; i < E; ++i) xs[i0 + i + ((i0 + i) >> 7)] = e[i];
            }
            __syncthreads();
            #pragma unroll
            for (int h = 0; h < 2; ++h) {
                const int t = warp + WARPS * h;
                const int k0 = 128 * ((lane & (lpr - 1)) + lpr * p) + 4 * t;
                const int l0 = k0 - kb;                        // inside the staged slice
                float e[4];
                #pragma unroll
                for (int j = 0; j < 4; ++j)      // l0 + j stays in l0's 128-block; chunks past the row read 0
                    e[j] = k0 < kpad ? xs[l0 + j + (l0 >> 7)] : 0.0f;
                float p01[4], p23[4];
                #pragma unroll
                for (int b = 0; b < 4; ++b) {
                    p01[b] = ((b & 1) ? -e[0] : e[0]) + ((b & 2) ? -e[1] : e[1]);
                    p23[b] = ((b & 1) ? -e[2] : e[2]) + ((b & 2) ? -e[3] : e[3]);
                }
                float* trow = table + ((p * 32 + t) * 16) * 32 + lane;
                #pragma unroll
                for (int m = 0; m < 16; ++m) trow[m * 32] = p01[m & 3] + p23[m >> 2];
            }
        }
    };

    const bool late_wait = prefetch && xstatic;
    if (prefetch) load_pass(0, 0);
    if (xstatic) build_table();
    if (dependent == 1 && !late_wait) grid_dependency_wait();
    if (!prefetch) load_pass(0, 0);
    if (!xstatic) build_table();
    __syncthreads();

    bool first = true;
    for (int64_t batch = 0; (gw + batch * total_warps) * rows_per_batch < N; ++batch) {
        float acc[U][4];
        #pragma unroll
        for (int u = 0; u < U; ++u)
            #pragma unroll
            for (int a = 0; a < 4; ++a) acc[u][a] = 0.0f;
        for (int p = 0; p < np; ++p) {
            if (batch > 0 || p > 0) load_pass(batch, p);
            const float* tp = table + p * PASS_FLOATS + lane;
            #pragma unroll
            for (int u = 0; u < U; ++u) {
                const uint32_t wq[4] = {v[u].x, v[u].y, v[u].z, v[u].w};
                #pragma unroll
                for (int q = 0; q < 4; ++q) {
                    #pragma unroll
                    for (int j = 0; j < 8; ++j) {
                        // nibble j of word q is group t = 8 q + j; entry m is
                        // m * 32 floats into the group's 512-float row.
                        const int t = 8 * q + j;
                        const uint32_t off = (4 * j >= 5 ? (wq[q] >> (4 * j - 5)) : (wq[q] << (5 - 4 * j))) & 0x1E0u;
                        acc[u][j & 3] += tp[t * 512 + off];
                    }
                }
            }
        }
        #pragma unroll
        for (int u = 0; u < U; ++u) {
            float s = (acc[u][0] + acc[u][1]) + (acc[u][2] + acc[u][3]);
            for (int off = lpr >> 1; off >= 1; off >>= 1) s += __shfl_xor_sync(0xffffffffu, s, off);
            acc[u][0] = s;
        }
        if (first && dependent == 1 && late_wait) grid_dependency_wait();
        first = false;
        if (li == 0) {
            #pragma unroll
            for (int u = 0; u < U; ++u) {
                const int64_t r = row_of(batch, u);
                if (r < N) y[r] = alpha[r] * acc[u][0];
            }
        }
    }
    if (dependent == 2) grid_dependency_wait();
}

}  // namespace bnn
