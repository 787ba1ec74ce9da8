// Ternary weights {-1, 0, +1} (BitNet b1.58) and their product with an int8
// activation vector.
//
// "Extreme Quantization: Binary, Ternary & 1-bit LLMs":
//  * Ternary Quantization, eq. (7): +1 where w > Delta, 0 where |w| <= Delta,
//    -1 where w < -Delta.
//  * BitNet b1.58, eq. (9): W_t = RoundClip(W / gamma, -1, 1) with
//    gamma = ||W||_1 / (n m), the mean |w| over the whole matrix.  Rounding
//    halves to even, RoundClip gives +-1 exactly where |w| > gamma / 2, which
//    is eq. (7) with Delta = gamma / 2.  gamma is summed in fp64; the
//    decision w > Delta is then taken exactly, as w >= (the smallest fp32
//    above Delta) in fp32 (fp32 and bf16 weights).
//  * BitNet: activations quantised to INT8.
// "First Principles: Why Binary Ops Can Be Exponentially Faster", the
// op-per-element table: a ternary weight adds, skips or subtracts.
//
// Packed layout: weight k of a row is the 2-bit code t + 1 (0, 1, 2) at bits
// 2(k mod 16) of word k / 16; a row holds ceil(K/16) words rounded up to a
// multiple of 4; positions past K hold code 1 (weight 0).
//
// Product.  With c = t + 1, sum_k t_k x_k = sum_k c_k x_k - sum_k x_k.  The
// byte lanes of word & (0x03030303 << 2j) hold the codes of weights j, 4+j,
// 8+j, 12+j of the word's 16 (times 4^j), so each mask meets a word of x
// holding the same four elements: the kernels stage x in shared memory with
// every group of 16 bytes transposed as a 4 x 4 byte matrix, and one dp4a
// then adds four products.  All arithmetic is in int32 and exact.
#pragma once

#include "common.cuh"

namespace bnn {

__host__ __device__ constexpr int64_t ternary_ld_words(int64_t K) { return ((K + 15) / 16 + 3) / 4 * 4; }

// ---------------------------------------------------------------------------
// gamma of eq. (9): per-row sums of |w| in fp64, then one block adds them in
// a fixed order (the same result on every run).
// ---------------------------------------------------------------------------

// One warp per row; U 16-byte vectors per lane in flight.
template <typename T, int U>
__global__ void __launch_bounds__(256)
ternary_abs_rowsum_kernel(const T* __restrict__ w, int64_t rows, int64_t K, int64_t ld_w, bool vec_ok,
                          double* __restrict__ rowsum) {
    constexpr int E = 16 / (int)sizeof(T);
    constexpr int CH = 32 * E;
    const int lane = threadIdx.x & 31;
    const int64_t row = (int64_t)blockIdx.x * (blockDim.x >> 5) + (threadIdx.x >> 5);
    grid_dependents_launch();                      // the gamma kernel may be scheduled now
    if (row >= rows) return;
    const T* wr = w + row * ld_w;
    const int64_t nchunks = (K + CH - 1) / CH;
    double s = 0.0;
    for (int64_t c0 = 0; c0 < nchunks; c0 += U) {
        float v[U][E];
        #pragma unroll
        for (int u = 0; u < U; ++u) {
            const int64_t base = (c0 + u) * CH + (int64_t)lane * E;
            if (vec_ok && base + E <= K) {
                const uint4 q = ldg_stream_v4(wr + base);
                const T* e = reinterpret_cast<const T*>(&q);
                #pragma unroll
                for (int i = 0; i < E; ++i) v[u][i] = to_float(e[i]);
            } else {
                #pragma unroll
                for (int i = 0; i < E; ++i) v[u][i] = (base + i < K) ? to_float(wr[base + i]) : 0.0f;
            }
        }
        #pragma unroll
        for (int u = 0; u < U; ++u) {
            #pragma unroll
            for (int i = 0; i < E; ++i) s += fabs((double)v[u][i]);
        }
    }
    #pragma unroll
    for (int off = 16; off >= 1; off >>= 1) s += __shfl_xor_sync(0xffffffffu, s, off);
    if (lane == 0) rowsum[row] = s;
}

// One block of 1024 threads: gamma = (sum of rowsum) / (rows * K) in fp64,
// written to *gamma_d and, rounded once, to *gamma_out (if given).  Launched
// as a programmatic dependent of the row-sum kernel: it waits for that grid
// before reading rowsum, and lets the pack kernel be scheduled at once.
__global__ void __launch_bounds__(1024)
ternary_gamma_kernel(const double* __restrict__ rowsum, int64_t rows, int64_t K, double* __restrict__ gamma_d,
                     float* __restrict__ gamma_out) {
    __shared__ double part[1024];
    grid_dependents_launch();
    grid_dependency_wait();
    double s = 0.0;
    for (int64_t r = threadIdx.x; r < rows; r += 1024) s += rowsum[r];
    part[threadIdx.x] = s;
    __syncthreads();
    for (int h = 512; h >= 1; h >>= 1) {
        if ((int)threadIdx.x < h) part[threadIdx.x] += part[threadIdx.x + h];
        __syncthreads();
    }
    if (threadIdx.x == 0) {
        const double g = part[0] / ((double)rows * (double)K);
        *gamma_d = g;
        if (gamma_out != nullptr) *gamma_out = (float)g;
    }
}

// ---------------------------------------------------------------------------
// Quantise and pack.  One warp per row.  A lane's 16-byte vector holds E
// elements = 2E code bits; the G = 16 / E lanes of one code word OR their
// bits together.  Delta is *gamma_src / 2 when gamma_src is given (eq. (9),
// gamma from the kernel above) and `delta` otherwise (eq. (7)).
// ---------------------------------------------------------------------------
// The decision w > Delta (Delta >= 0 in fp64) for an fp32 w, taken exactly in
// fp32: w > Delta  <=>  w >= up, with up the smallest fp32 value above Delta
// (NaN when there is none, Delta = +inf, so that nothing compares true).
__device__ __forceinline__ float fp32_above(double delta) {
    if (!(delta < (double)INFINITY)) return __int_as_float(0x7fc00000);
    float f = __double2float_ru(delta);               // smallest fp32 >= delta (inf past FLT_MAX)
    if ((double)f == delta) f = nextafterf(f, INFINITY);
    return f;
}

// Launched after the gamma kernel as its programmatic dependent (eq. (9), or
// when gamma is reported): the first weight vectors are loaded before the
// wait for that grid, which must end before gamma is read.  Elements past K
// are loaded as 0.0, which quantises to code 1 (up > 0 or NaN), the pad code.
template <typename T, int U>
__global__ void __launch_bounds__(256)
pack_ternary_kernel(const T* __restrict__ w, int64_t rows, int64_t K, int64_t ld_w, bool vec_ok,
                    const double* __restrict__ gamma_src, double delta, uint32_t* __restrict__ codes,
                    int64_t ldq) {
    constexpr int E = 16 / (int)sizeof(T);
    constexpr int G = 16 / E;                      // lanes per code word
    constexpr int CH = 32 * E;                     // elements per warp chunk
    const int lane = threadIdx.x & 31;
    const int64_t row = (int64_t)blockIdx.x * (blockDim.x >> 5) + (threadIdx.x >> 5);
    const bool active = row < rows;
    const T* wr = w + (active ? row : 0) * ld_w;
    uint32_t* qr = codes + (active ? row : 0) * ldq;
    const int64_t nw = ternary_ld_words(K);
    const int64_t nchunks = (nw * 16 + CH - 1) / CH;
    float v[U][E];
    auto load = [&](int64_t c0) {
        #pragma unroll
        for (int u = 0; u < U; ++u) {
            const int64_t base = (c0 + u) * CH + (int64_t)lane * E;
            if (vec_ok && base + E <= K) {
                const uint4 q = ldg_stream_v4(wr + base);
                const T* e = reinterpret_cast<const T*>(&q);
                #pragma unroll
                for (int i = 0; i < E; ++i) v[u][i] = to_float(e[i]);
            } else {
                #pragma unroll
                for (int i = 0; i < E; ++i) v[u][i] = (base + i < K) ? to_float(wr[base + i]) : 0.0f;
            }
        }
    };
    if (active) load(0);
    grid_dependency_wait();
    if (!active) return;
    const float up = fp32_above(gamma_src != nullptr ? 0.5 * *gamma_src : delta);
    const float dn = -up;
    for (int64_t c0 = 0; c0 < nchunks; c0 += U) {
        if (c0 > 0) load(c0);
        #pragma unroll
        for (int u = 0; u < U; ++u) {
            const int64_t chunk = c0 + u;
            if (chunk >= nchunks) break;
            uint32_t bits = 0;
            #pragma unroll
            for (int i = 0; i < E; ++i) {
                const uint32_t c = v[u][i] >= up ? 2u : (v[u][i] <= dn ? 0u : 1u);   // NaN -> 1 (weight 0)
                bits += c << (2 * i);
            }
            bits <<= 2 * E * (lane % G);
            #pragma unroll
            for (int off = 1; off < G; off <<= 1) bits |= __shfl_xor_sync(0xffffffffu, bits, off);
            const int64_t wi = chunk * (CH / 16) + lane / G;
            if ((lane % G) == 0 && wi < nw) qr[wi] = bits;
        }
    }
}

// ---------------------------------------------------------------------------
// GEMV: y[n] = sum_k t_nk x_k, int8 x, exact int32; optionally
// y_f32[n] = fp32(fp32(w_scale * x_scale) * fp32(acc)).
//
// x is staged in shared memory, every 16 elements (one code word) transposed
// as a 4 x 4 byte matrix: word j of group g holds x[16g+j], x[16g+4+j],
// x[16g+8+j], x[16g+12+j].  Group g = 4c + q (chunk c of 16 bytes of codes,
// word q) goes to words 4 (q * nch + c) .. + 3, so the 32 lanes of a warp,
// reading 32 consecutive chunks, read 512 contiguous bytes.
//
// Per code word w, the bytes of w & 0x03030303 and w & 0x0C0C0C0C hold the
// codes that meet words 0 and 1 of the staged group (the second scaled by
// 4), and the same masks of w >> 4 those of words 2 and 3.  dp4a (unsigned
// codes, signed x) adds four products; with one accumulator for each scale,
// the lane total is acc0 + acc1 / 4 (exact: acc1 is a multiple of 4).  A
// lane also adds up its own x elements once: the row total is
// sum c x - sum x, one warp reduction.
// ---------------------------------------------------------------------------
namespace tgv {
constexpr int64_t MAX_WORDS = 6144;        // staged x = 16 bytes per code word: 96 KiB (K <= 98304)
}  // namespace tgv

__device__ __forceinline__ int dp4a_us(uint32_t a, uint32_t b, int c) {
    int d;
    asm("dp4a.u32.s32 %0, %1, %2, %3;" : "=r"(d) : "r"(a), "r"(b), "r"(c));
    return d;
}

__device__ __forceinline__ void stage_x_transposed(const int8_t* __restrict__ x, int K, int nw, bool vec_ok,
                                                   uint32_t* xs) {
    const int nch = nw / 4;
    for (int g = threadIdx.x; g < nw; g += blockDim.x) {
        uint32_t a[4];
        if (vec_ok && 16 * g + 16 <= K) {
            const uint4 q = *reinterpret_cast<const uint4*>(x + 16 * g);
            a[0] = q.x; a[1] = q.y; a[2] = q.z; a[3] = q.w;
        } else {
            #pragma unroll
            for (int i = 0; i < 4; ++i) {
                uint32_t wv = 0;
                #pragma unroll
                for (int b = 0; b < 4; ++b) {
                    const int k = 16 * g + 4 * i + b;
                    const uint32_t byte = k < K ? (uint32_t)(uint8_t)x[k] : 0u;
                    wv |= byte << (8 * b);
                }
                a[i] = wv;
            }
        }
        const uint32_t t0 = __byte_perm(a[0], a[1], 0x5140);   // a0.b0 a1.b0 a0.b1 a1.b1
        const uint32_t t1 = __byte_perm(a[2], a[3], 0x5140);
        const uint32_t t2 = __byte_perm(a[0], a[1], 0x7362);   // a0.b2 a1.b2 a0.b3 a1.b3
        const uint32_t t3 = __byte_perm(a[2], a[3], 0x7362);
        *reinterpret_cast<uint4*>(xs + 4 * ((g & 3) * nch + (g >> 2))) =
            make_uint4(__byte_perm(t0, t1, 0x5410), __byte_perm(t0, t1, 0x7632), __byte_perm(t2, t3, 0x5410),
                       __byte_perm(t2, t3, 0x7632));
    }
    __syncthreads();
}

// One chunk (4 code words) of one row against its 4 staged x groups X[0..3].
__device__ __forceinline__ void ternary_chunk(const uint4 wc, const uint4 (&X)[4], int (&acc)[2]) {
    const uint32_t wq[4] = {wc.x, wc.y, wc.z, wc.w};
    #pragma unroll
    for (int q = 0; q < 4; ++q) {
        const uint32_t hi = wq[q] >> 4;
        acc[0] = dp4a_us(wq[q] & 0x03030303u, X[q].x, acc[0]);
        acc[1] = dp4a_us(wq[q] & 0x0C0C0C0Cu, X[q].y, acc[1]);
        acc[0] = dp4a_us(hi & 0x03030303u, X[q].z, acc[0]);
        acc[1] = dp4a_us(hi & 0x0C0C0C0Cu, X[q].w, acc[1]);
    }
}

__device__ __forceinline__ int xsum_chunk(const uint4 (&X)[4], int s) {
    #pragma unroll
    for (int q = 0; q < 4; ++q) {
        s = __dp4a((int)X[q].x, 0x01010101, s);
        s = __dp4a((int)X[q].y, 0x01010101, s);
        s = __dp4a((int)X[q].z, 0x01010101, s);
        s = __dp4a((int)X[q].w, 0x01010101, s);
    }
    return s;
}

__device__ __forceinline__ void load_x_chunk(const uint32_t* xs, int nch, int c, uint4 (&X)[4]) {
    #pragma unroll
    for (int q = 0; q < 4; ++q) X[q] = *reinterpret_cast<const uint4*>(xs + 4 * (q * nch + c));
}

__device__ __forceinline__ int lane_total(const int (&acc)[2], int xsum) {
    return acc[0] + (acc[1] >> 2) - xsum;
}

// TH threads per block; a warp owns U rows.  Lane l reads the 16-byte chunks
// l, l + 32, ... of each row (a warp-wide load is 512 contiguous bytes of one
// row) and P chunks per row are in flight before any is used.  Programmatic
// dependent launch as the XNOR GEMV: static weights are loaded before the
// wait for the previous grid, static inputs staged before it too.  The
// launcher picks U per dependency mode (independent steps: U = 4, 344 blocks
// at N = 11008; a dependent chain: U = 8, fewer and fuller blocks).
template <int TH, int U, int P>
__global__ void __launch_bounds__(TH)
ternary_gemv_i8_kernel(const uint32_t* __restrict__ Q, int64_t ldq, const int8_t* __restrict__ x, int N, int K,
                       int nw, bool x_vec, const float* __restrict__ w_scale, const float* __restrict__ x_scale,
                       int32_t* __restrict__ y_i32, float* __restrict__ y_f32, int prefetch, int xstatic,
                       int dependent) {
    constexpr int WARPS = TH / 32;
    extern __shared__ __align__(16) uint32_t txs[];
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int row0 = (blockIdx.x * WARPS + warp) * U;
    const int nch = nw / 4;                               // 16-byte chunks per row
    const int passes = (nch + 32 * P - 1) / (32 * P);
    grid_dependents_launch();

    uint4 v[P][U];
    auto load_pass = [&](int sp) {
        #pragma unroll
        for (int p = 0; p < P; ++p) {
            const int c = lane + 32 * (sp * P + p);
            #pragma unroll
            for (int u = 0; u < U; ++u) {
                const int r = row0 + u;
                v[p][u] = (r < N && c < nch) ? ldg_stream_v4(Q + (int64_t)r * ldq + 4 * c)
                                             : make_uint4(0u, 0u, 0u, 0u);
            }
        }
    };
    // w_scale belongs to the weights (read with them), x_scale to x.
    float scale = 1.0f, wsc = 1.0f;
    auto load_weights = [&]() {
        load_pass(0);
        if (y_f32 != nullptr && w_scale != nullptr) wsc = *w_scale;
    };
    auto stage = [&]() {
        stage_x_transposed(x, K, nw, x_vec, txs);
        if (y_f32 != nullptr) scale = wsc * (x_scale != nullptr ? *x_scale : 1.0f);
    };
    const bool late_wait = prefetch && xstatic;
    if (prefetch) load_weights();
    if (xstatic) stage();
    if (dependent == 1 && !late_wait) grid_dependency_wait();
    if (!prefetch) load_weights();
    if (!xstatic) stage();

    int acc[U][2];
    #pragma unroll
    for (int u = 0; u < U; ++u) acc[u][0] = acc[u][1] = 0;
    int xsum = 0;
    for (int sp = 0; sp < passes; ++sp) {
        if (sp > 0) load_pass(sp);
        #pragma unroll
        for (int p = 0; p < P; ++p) {
            const int c = lane + 32 * (sp * P + p);
            if (c < nch) {
                uint4 X[4];
                load_x_chunk(txs, nch, c, X);
                xsum = xsum_chunk(X, xsum);
                #pragma unroll
                for (int u = 0; u < U; ++u) ternary_chunk(v[p][u], X, acc[u]);
            }
        }
    }
    int tot[U];
    #pragma unroll
    for (int u = 0; u < U; ++u) tot[u] = __reduce_add_sync(0xffffffffu, lane_total(acc[u], xsum));
    if (dependent == 1 && late_wait) grid_dependency_wait();
    if (lane == 0) {
        #pragma unroll
        for (int u = 0; u < U; ++u) {
            const int r = row0 + u;
            if (r < N) {
                if (y_i32 != nullptr) y_i32[r] = tot[u];
                if (y_f32 != nullptr) y_f32[r] = scale * (float)tot[u];
            }
        }
    }
    if (dependent == 2) exit_after_previous_grid();
}

}  // namespace bnn
