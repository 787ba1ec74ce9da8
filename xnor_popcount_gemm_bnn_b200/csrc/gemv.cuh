// Batch-1 binary GEMV: y[n] = K - 2 * popcount(W[n, :] XOR pack(sign(x))).
//
// "First Principles: Why Binary Ops Can Be Exponentially Faster", "Bandwidth
// math": a batch-1 y = Wx moves about MN/8 bytes once W is packed, so the
// kernel is bound by streaming the packed W from HBM.  "Extreme Quantization:
// Binary, Ternary & 1-bit LLMs", eq. (4) (x is binarised too) and eq. (6).
//
// Design (sm_100a):
//  * Each CTA packs the real x into shared memory itself (one ballot per
//    32 elements; x is a few KB and stays in L2), so the whole GEMV is one
//    launch.
//  * The packed rows are read as 16-byte non-allocating vectors, LPR lanes per
//    row (LPR = 32 when a row is >= 512 bytes, i.e. K >= 4096), so a warp-wide
//    load is one contiguous row segment.  Each warp issues the loads of its U
//    row groups before using any of them; all of W is in flight at once.
//  * Row sums: redux.sync (one instruction) when LPR = 32, else a shuffle tree.
//  * Launched with programmatic dependent launch: the grid may start while
//    the previous kernel on the stream finishes, and waits for it
//    (griddepcontrol.wait) before reading x and before writing y.  When the
//    caller declares the weights static (nothing still in flight on the stream
//    writes W or alpha), the W and alpha loads are issued before that wait, so
//    the weight stream of consecutive GEMVs runs back to back.
#pragma once

#include "common.cuh"

namespace bnn {
namespace gemv {
// Block shape of the general kernel: 512 threads x 2 row groups per warp.
// (The one-chunk-per-lane kernel below takes its shape as template
// parameters, chosen per dependency mode by the launcher.)
constexpr int THREADS = 512;
constexpr int WARPS = THREADS / 32;
constexpr int U = 2;   // row groups per warp

}  // namespace gemv

// Packs the real vector x (K elements, zero past K up to kw words) into xs[]
// (shared memory), one bit per element, bit 1 for x < 0.  VEC: x is 16-byte
// aligned, so each thread loads whole 16-byte vectors (8 bf16 or 4 fp32);
// all of a thread's loads are issued before any bit is assembled, and the
// E bits of a vector are OR-combined across the 32/E lanes of a word.
template <typename XT, bool VEC>
__device__ __forceinline__ void gemv_pack_x(const XT* __restrict__ x, int K, int kw, uint32_t* xs) {
    using namespace gemv;
    const int lane = threadIdx.x & 31;
    if constexpr (VEC) {
        constexpr int E = 16 / (int)sizeof(XT);       // elements per vector
        constexpr int G = 32 / E;                     // lanes per packed word
        constexpr int VB = 2;                         // vectors per thread per batch
        const int nvec = kw * 32 / E;                 // vectors covering the padded row
        for (int v0 = 0; v0 < nvec; v0 += THREADS * VB) {
            float e[VB][E];
            #pragma unroll
            for (int b = 0; b < VB; ++b) {
                const int vi = v0 + b * THREADS + (int)threadIdx.x;
                const int base = vi * E;
                if (base + E <= K) {
                    const uint4 q = *reinterpret_cast<const uint4*>(x + base);
                    const XT* el = reinterpret_cast<const XT*>(&q);
                    #pragma unroll
                    for (int i = 0; i < E; ++i) e[b][i] = to_float(el[i]);
                } else {
                    #pragma unroll
                    for (int i = 0; i < E; ++i) e[b][i] = (vi < nvec && base + i < K) ? to_float(x[base + i]) : 0.0f;
                }
            }
            #pragma unroll
            for (int b = 0; b < VB; ++b) {
                const int vi = v0 + b * THREADS + (int)threadIdx.x;
                uint32_t bits = 0;
                #pragma unroll
                for (int i = 0; i < E; ++i) bits |= neg_bit(e[b][i]) << i;
                bits <<= E * (lane % G);
                #pragma unroll
                for (int off = 1; off < G; off <<= 1) bits |= __shfl_xor_sync(0xffffffffu, bits, off);
                if ((lane % G) == 0 && vi < nvec) xs[vi / G] = bits;
            }
        }
    } else {
        constexpr int XB = 8;                         // words per warp per batch, loads first
        const int warp = threadIdx.x >> 5;
        for (int wd0 = warp; wd0 < kw; wd0 += WARPS * XB) {
            float xv[XB];
            #pragma unroll
            for (int j = 0; j < XB; ++j) {
                const int wd = wd0 + WARPS * j;
                const int e = 32 * wd + lane;
                xv[j] = (wd < kw && e < K) ? to_float(x[e]) : 0.0f;
            }
            #pragma unroll
            for (int j = 0; j < XB; ++j) {
                const int wd = wd0 + WARPS * j;
                const uint32_t word = __ballot_sync(0xffffffffu, xv[j] < 0.0f);
                if (lane == 0 && wd < kw) xs[wd] = word;
            }
        }
    }
}

// Fast path for rows of 68..128 words (LPR = 32, one 16-byte chunk per lane,
// K <= 4096) and a 16-byte aligned x: each lane owns one chunk of U rows, the
// x pack is one vector per thread per round (E elements; 32/E lanes OR their
// bits into a word).  Measured about 20% shorter steps than the generic
// kernel in dependent back-to-back launches.
//
// The block shape (TH threads, U rows per warp) is a template parameter: the
// launcher picks it per dependency mode (see row128_shape in the library).
template <typename XT, int TH, int U>
__global__ void __launch_bounds__(TH)
xnor_gemv_row128_kernel(const uint32_t* __restrict__ W, int64_t ldw, const XT* __restrict__ x, int N, int K,
                        int kw, const float* __restrict__ alpha, int32_t* __restrict__ y_i32,
                        float* __restrict__ y_f32, int prefetch, int xstatic, int dependent) {
    constexpr int THREADS = TH;
    constexpr int WARPS = TH / 32;
    constexpr int E = 16 / (int)sizeof(XT);           // elements per 16-byte vector
    constexpr int G = 32 / E;                         // lanes per packed word
    extern __shared__ __align__(16) uint32_t xs[];
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int64_t gw = (int64_t)blockIdx.x * WARPS + warp;
    int rows[U];
    #pragma unroll
    for (int u = 0; u < U; ++u) rows[u] = (int)(gw * U + u);
    grid_dependents_launch();
    const int nch = kw / 4;
    uint4 v[U];
    float al[U];                                      // alpha of the rows this lane stores (lane 0)
    // The weights and their per-row scale, read together.
    auto load_w = [&]() {
        #pragma unroll
        for (int u = 0; u < U; ++u) {
            v[u] = (rows[u] < N && lane < nch) ? ldg_stream_v4(W + (int64_t)rows[u] * ldw + 4 * lane)
                                               : make_uint4(0u, 0u, 0u, 0u);
            al[u] = (lane == 0 && y_f32 != nullptr && rows[u] < N) ? alpha[rows[u]] : 0.0f;
        }
    };
    auto pack_x = [&]() {
        const int nfull = K / E;                      // whole vectors inside x
        const int nvec = kw * (32 / E);               // vectors covering the padded row
        // The trip count is block-uniform (c0 steps over whole blocks), so
        // every lane of a warp reaches the full-mask shuffle together even
        // when nvec is not a multiple of 32; lanes past nvec carry zeros.
        for (int c0 = 0; c0 < nvec; c0 += THREADS) {
            const int c = c0 + (int)threadIdx.x;
            uint4 q = make_uint4(0u, 0u, 0u, 0u);
            if (c < nfull) q = *reinterpret_cast<const uint4*>(x + E * c);
            const XT* e = reinterpret_cast<const XT*>(&q);
            uint32_t b = 0;
            #pragma unroll
            for (int i = 0; i < E; ++i) b |= neg_bit(to_float(e[i])) << i;
            if (c == nfull && c < nvec) {             // the partial last vector, if any
                b = 0;
                for (int i = 0; i < K - E * c; ++i) b |= neg_bit(to_float(x[E * c + i])) << i;
            }
            b <<= E * (c & (G - 1));
            #pragma unroll
            for (int off = 1; off < G; off <<= 1) b |= __shfl_xor_sync(0xffffffffu, b, off);
            if ((c & (G - 1)) == 0 && c < nvec) xs[c / G] = b;
        }
        __syncthreads();
    };
    // Everything that reads only static data runs before the dependency wait:
    // the weight stream (prefetch), the x pack (xstatic), and with both the
    // whole product, so that only the store of y waits.
    if (prefetch) load_w();
    if (xstatic) pack_x();
    const bool late_wait = prefetch && xstatic;
    if (dependent == 1 && !late_wait) grid_dependency_wait();
    if (!prefetch) load_w();
    if (!xstatic) pack_x();
    const uint4 xq = lane < nch ? *reinterpret_cast<const uint4*>(xs + 4 * lane) : make_uint4(0u, 0u, 0u, 0u);
    uint32_t d[U];
    #pragma unroll
    for (int u = 0; u < U; ++u) d[u] = __reduce_add_sync(0xffffffffu, popc_xor4(v[u], xq));
    if (dependent == 1 && late_wait) grid_dependency_wait();
    #pragma unroll
    for (int u = 0; u < U; ++u) {
        const int r = rows[u];
        if (lane == 0 && r < N) {
            const int32_t sv = K - 2 * (int32_t)d[u];
            if (y_i32 != nullptr) y_i32[r] = sv;
            if (y_f32 != nullptr) y_f32[r] = al[u] * (float)sv;
        }
    }
    // dependent == 2: the call touches nothing that work in flight uses; its
    // completion must still imply the previous grid's (stream order stays
    // transitive), which one block waiting before it exits is enough for.
    if (dependent == 2) exit_after_previous_grid();
}

// SINGLE: every row fits in one warp-wide pass (nchunks <= LPR).
// PREFETCH: issue the W loads before the programmatic-launch wait.
// VEC: x is 16-byte aligned (vector loads for the x pack).
template <typename XT, int LPR, bool SINGLE, bool PREFETCH, bool VEC>
__global__ void __launch_bounds__(gemv::THREADS)
xnor_gemv_kernel(const uint32_t* __restrict__ W, int64_t ldw, const XT* __restrict__ x, int N,
                 int K, int kw, const float* __restrict__ alpha, int32_t* __restrict__ y_i32,
                 float* __restrict__ y_f32, int dependent) {
    using namespace gemv;
    constexpr int RPI = 32 / LPR;  // rows per warp-wide load
    extern __shared__ __align__(16) uint32_t xs[];
    const int warp = threadIdx.x >> 5;
    const int lane = threadIdx.x & 31;
    const int nchunks = kw / 4;                       // 16-byte chunks per row
    const int sub = lane / LPR;                       // row within a warp-wide load
    const int li = lane % LPR;                        // lane within the row
    const int row0 = (blockIdx.x * WARPS + warp) * U * RPI + sub;   // rows row0 + u * RPI

    // Let the next kernel on the stream start its own prologue now; it waits
    // for this grid to finish before it touches anything this grid writes.
    grid_dependents_launch();

    uint4 v[U];
    float al[U];                                      // alpha of the rows this lane stores (li == 0)
    auto load_pass = [&](int t) {
        const int c = li + LPR * t;
        #pragma unroll
        for (int u = 0; u < U; ++u) {
            const int r = row0 + u * RPI;
            v[u] = (r < N && c < nchunks) ? ldg_stream_v4(W + (int64_t)r * ldw + 4 * c)
                                          : make_uint4(0u, 0u, 0u, 0u);
        }
    };
    auto load_alpha = [&]() {
        #pragma unroll
        for (int u = 0; u < U; ++u) {
            const int r = row0 + u * RPI;
            al[u] = (li == 0 && y_f32 != nullptr && r < N) ? alpha[r] : 0.0f;
        }
    };

    // The weight stream does not depend on x.  With static weights it starts
    // before the dependency wait (overlapping the previous kernel's tail);
    // otherwise right after it, still ahead of the x loads.
    // `dependent` is always 1 from the host.  Keeping the wait behind a
    // run-time branch puts it in its own basic block, so the instruction
    // scheduler cannot hoist it above the weight loads issued before it.
    if constexpr (PREFETCH) {
        load_pass(0);
        load_alpha();
    }
    if (dependent) grid_dependency_wait();
    if constexpr (!PREFETCH) {
        load_pass(0);
        load_alpha();
    }

    gemv_pack_x<XT, VEC>(x, K, kw, xs);
    __syncthreads();

    uint32_t d[U];
    if constexpr (SINGLE) {
        const uint4 xq = li < nchunks ? *reinterpret_cast<const uint4*>(xs + 4 * li)
                                      : make_uint4(0u, 0u, 0u, 0u);
        #pragma unroll
        for (int u = 0; u < U; ++u) d[u] = popc_xor4(v[u], xq);
    } else {
        #pragma unroll
        for (int u = 0; u < U; ++u) d[u] = 0u;
        const int passes = (nchunks + LPR - 1) / LPR;
        for (int t = 0; t < passes; ++t) {
            if (t > 0) load_pass(t);
            const int c = li + LPR * t;
            const uint4 xq = (c < nchunks) ? *reinterpret_cast<const uint4*>(xs + 4 * c)
                                           : make_uint4(0u, 0u, 0u, 0u);
            #pragma unroll
            for (int u = 0; u < U; ++u) d[u] += popc_xor4(v[u], xq);
        }
    }

    #pragma unroll
    for (int u = 0; u < U; ++u) {
        uint32_t dd = d[u];
        if constexpr (LPR == 32) {
            dd = __reduce_add_sync(0xffffffffu, dd);
        } else {
            #pragma unroll
            for (int off = LPR / 2; off >= 1; off >>= 1) dd += __shfl_xor_sync(0xffffffffu, dd, off);
        }
        const int r = row0 + u * RPI;
        if (li == 0 && r < N) {
            const int32_t sv = K - 2 * (int32_t)dd;
            if (y_i32 != nullptr) y_i32[r] = sv;
            if (y_f32 != nullptr) y_f32[r] = al[u] * (float)sv;
        }
    }
}

}  // namespace bnn
