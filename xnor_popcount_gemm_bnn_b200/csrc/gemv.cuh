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
//    row groups before using any of them, keeping U * 512 bytes per warp in
//    flight.
//  * Row sums: redux.sync (one instruction) when LPR = 32, else a shuffle tree.
//  * Launched with programmatic dependent launch: the grid may start while
//    the previous kernel on the stream finishes, and waits for it
//    (griddepcontrol.wait) before reading x or alpha and before writing y.
//    When the caller declares the weights static (nothing still in flight on
//    the stream writes W), the W loads are issued before that wait, so the
//    weight stream of consecutive GEMVs runs back to back.
#pragma once

#include "common.cuh"

namespace bnn {
namespace gemv {
constexpr int THREADS = 256;
constexpr int WARPS = THREADS / 32;
constexpr int U = 4;   // row groups per warp
}  // namespace gemv

template <typename XT, int LPR>
__global__ void __launch_bounds__(gemv::THREADS)
xnor_gemv_kernel(const uint32_t* __restrict__ W, int64_t ldw, const XT* __restrict__ x, int N,
                 int K, int kw, const float* __restrict__ alpha, int32_t* __restrict__ y_i32,
                 float* __restrict__ y_f32, bool weights_static) {
    using namespace gemv;
    constexpr int RPI = 32 / LPR;  // rows per warp-wide load
    constexpr int XB = 16;         // x words packed per warp per batch (all loads in flight)
    extern __shared__ __align__(16) uint32_t xs[];
    const int warp = threadIdx.x >> 5;
    const int lane = threadIdx.x & 31;
    const int nchunks = kw / 4;                       // 16-byte chunks per row
    const int64_t gw = (int64_t)blockIdx.x * WARPS + warp;
    const int sub = lane / LPR;                       // row within a warp-wide load
    const int li = lane % LPR;                        // lane within the row
    int rows[U];
    #pragma unroll
    for (int u = 0; u < U; ++u) rows[u] = (int)((gw * U + u) * RPI + sub);

    // Let the next kernel on the stream start its own prologue now; it waits
    // for this grid to finish before it touches anything this grid writes.
    grid_dependents_launch();

    uint4 v[U];
    auto load_pass = [&](int t) {
        const int c = li + LPR * t;
        #pragma unroll
        for (int u = 0; u < U; ++u)
            v[u] = (rows[u] < N && c < nchunks)
                       ? ldg_stream_v4(W + (int64_t)rows[u] * ldw + 4 * c)
                       : make_uint4(0u, 0u, 0u, 0u);
    };

    // The weight stream does not depend on x.  With static weights it starts
    // before the dependency wait (overlapping the previous kernel's tail);
    // otherwise right after it, still ahead of the x loads.
    if (weights_static) load_pass(0);
    grid_dependency_wait();
    if (!weights_static) load_pass(0);

    // Pack x into shared memory: word wd <- ballot over elements 32*wd + lane.
    // XB words per warp per batch, all loads issued before the first ballot.
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
    __syncthreads();

    uint32_t d[U];
    #pragma unroll
    for (int u = 0; u < U; ++u) d[u] = 0u;
    const int passes = (nchunks + LPR - 1) / LPR;
    for (int t = 0; t < passes; ++t) {
        if (t > 0) load_pass(t);
        const int c = li + LPR * t;
        const uint4 xv = (c < nchunks) ? *reinterpret_cast<const uint4*>(xs + 4 * c)
                                       : make_uint4(0u, 0u, 0u, 0u);
        #pragma unroll
        for (int u = 0; u < U; ++u) d[u] += popc_xor4(v[u], xv);
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
        const int r = rows[u];
        if (li == 0 && r < N) {
            const int32_t s = K - 2 * (int32_t)dd;
            if (y_i32 != nullptr) y_i32[r] = s;
            if (y_f32 != nullptr) y_f32[r] = alpha[r] * (float)s;
        }
    }
}

}  // namespace bnn
