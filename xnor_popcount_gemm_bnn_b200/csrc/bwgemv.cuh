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
// Each warp issues the loads of U rows before the table is built (the weight
// stream overlaps it), sums each row on 4 accumulators per lane, and adds the
// lanes of a row with a butterfly of shuffles -- no block barrier after the
// table.
//
// Table layout (per pass, 64 KiB, at a 32 KiB-aligned shared address).  The
// entries a lane can ever look up (the groups of its own chunks) sit in bank
// `lane`, so the 32 lookups of a warp never conflict, whatever the nibbles.
// Groups come in pairs (nibbles 2P and 2P+1 of the lane's chunk): the even
// group's entry m is at byte (m << 7) | (P << 11), the odd group's at
// 32768 | (P << 7) | (m << 11), plus 4 * lane.  One shift of a packed word
// then puts nibble 2P at bits 7..10 and nibble 2P+1 at bits 11..14, and each
// lookup address is a single LOP3, (v & mask) | base, with the group's offset
// as the load's immediate: per two lookups one shift, two LOP3, two loads
// and two adds.
//
// Launched with programmatic dependent launch, like the XNOR GEMV: with static
// weights the first W and alpha loads precede the wait for the previous grid,
// with static inputs the table and the product do too (only the store waits),
// and with all three flags only block 0 waits, before it exits.
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
constexpr int PASS_BYTES = 32 * 16 * 32 * 4;
// The slice of x one pass reads (32 chunks x 128 elements), staged as fp32
// with one pad float after every 128 elements, so that lanes reading 128
// elements apart fall on distinct banks.  It sits below the table.
constexpr int XS_FLOATS = 4096 + 32;
constexpr int TABLE_ALIGN = 32768;
// The x slice, the padding up to the 32 KiB-aligned table (the dynamic
// window starts below 32 KiB - x slice, checked in the kernel), the table.
__host__ __device__ constexpr int smem_bytes(int kw) { return TABLE_ALIGN + passes(kw) * PASS_BYTES; }

}  // namespace bwg

// Two lookups of the pair P: v holds nibble 2P at bits 7..10 and nibble 2P+1
// at bits 11..14; lb = table + pass offset + 4 * lane (zero in bits 7..14).
template <int P>
__device__ __forceinline__ void bw_lookup_pair(uint32_t v, uint32_t lb, float& acc_even, float& acc_odd) {
    const uint32_t re = (v & 0x780u) | lb, ro = (v & 0x7800u) | lb;
    float e, o;
    asm volatile("ld.shared.f32 %0, [%1+%2];" : "=f"(e) : "r"(re), "n"(P << 11));
    asm volatile("ld.shared.f32 %0, [%1+%2];" : "=f"(o) : "r"(ro), "n"(32768 + (P << 7)));
    acc_even += e;
    acc_odd += o;
}

// The 8 nibbles of word Q of the lane's chunk (groups 8Q .. 8Q+7); nibble j
// goes to accumulator j mod 4.
template <int Q>
__device__ __forceinline__ void bw_lookup_word(uint32_t w, uint32_t lb, float (&acc)[4]) {
    bw_lookup_pair<4 * Q + 0>(w << 7, lb, acc[0], acc[1]);
    bw_lookup_pair<4 * Q + 1>(w >> 1, lb, acc[2], acc[3]);
    bw_lookup_pair<4 * Q + 2>(w >> 9, lb, acc[0], acc[1]);
    bw_lookup_pair<4 * Q + 3>(w >> 17, lb, acc[2], acc[3]);
}

__device__ __forceinline__ uint32_t dynamic_smem_size() {
    uint32_t r;
    asm("mov.u32 %0, %%dynamic_smem_size;" : "=r"(r));
    return r;
}

template <typename XT>
__global__ void __launch_bounds__(bwg::THREADS, 2)
bw_gemv_kernel(const uint32_t* __restrict__ W, int64_t ldw, const XT* __restrict__ x, int N, int K, int kw,
               const float* __restrict__ alpha, float* __restrict__ y, int prefetch, int xstatic, int dependent) {
    using namespace bwg;
    extern __shared__ __align__(16) float bw_smem[];
    const int np = passes(kw);
    // x slice at the start of the window, the table at the first 32 KiB
    // boundary above it.  The launcher requests TABLE_ALIGN + np passes;
    // a window that starts too high for that is reported, never overrun.
    const uint32_t s0 = smem_u32(bw_smem);
    const uint32_t t0 = (s0 + (uint32_t)(XS_FLOATS * 4) + (TABLE_ALIGN - 1)) & ~(uint32_t)(TABLE_ALIGN - 1);
    if (t0 - s0 + (uint32_t)np * PASS_BYTES > dynamic_smem_size()) {
        if (threadIdx.x == 0) flag_device_error(BNN_ERR_UNSUPPORTED);
        grid_dependency_wait();
        return;
    }
    float* xs = bw_smem;
    char* table = reinterpret_cast<char*>(bw_smem) + (t0 - s0);
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int nch = kw / 4;                                   // 16-byte chunks per row
    int lpr = 1;                                              // lanes per row: a power of two >= min(nch, 32)
    while (lpr < 32 && lpr < nch) lpr <<= 1;
    const int rpi = 32 / lpr;                                 // rows per warp-wide load
    const int li = lane & (lpr - 1), sub = lane / lpr;
    const int rows_per_batch = U * rpi;                       // rows of one warp per batch
    const int total_warps = (int)gridDim.x * WARPS;
    const int gw = (int)blockIdx.x * WARPS + warp;
    grid_dependents_launch();

    uint4 v[U];
    float al[U];                                              // alpha of the rows this lane stores (li == 0)
    // Rows of a batch: row0 + u * rpi for row0 = first row of the warp's batch + sub.
    // The first pass also reads the rows' alpha: the weights and their scale
    // are read together.
    const int64_t row_step = (int64_t)rpi * ldw;               // words between the rows of one load pass
    auto load_pass = [&](int row0, int p) {
        const int c = li + lpr * p;
        const uint32_t* wp = W + (int64_t)row0 * ldw + 4 * c;
        #pragma unroll
        for (int u = 0; u < U; ++u) {
            v[u] = (row0 + u * rpi < N && c < nch) ? ldg_stream_v4(wp) : make_uint4(0u, 0u, 0u, 0u);
            wp += row_step;
            if (p == 0) al[u] = (li == 0 && row0 + u * rpi < N) ? alpha[row0 + u * rpi] : 0.0f;
        }
    };
    // Per pass: the pass's slice of x -> shared fp32 (coalesced 16-byte loads
    // when x is aligned), then that pass's table: entry (t, m) of lane l =
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
            char* tp = table + p * PASS_BYTES + 4 * lane;
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
                // Entry m of an even group at (m << 7) | (P << 11), of an odd
                // group at 32768 | (P << 7) | (m << 11): one base per group and
                // compile-time offsets per entry.  (t's parity is warp-uniform.)
                const uint32_t P = (uint32_t)t >> 1;
                if (t & 1) {
                    float* ge = reinterpret_cast<float*>(tp + (32768u | (P << 7)));
                    #pragma unroll
                    for (int m = 0; m < 16; ++m) ge[m * 512] = p01[m & 3] + p23[m >> 2];
                } else {
                    float* ge = reinterpret_cast<float*>(tp + (P << 11));
                    #pragma unroll
                    for (int m = 0; m < 16; ++m) ge[m * 32] = p01[m & 3] + p23[m >> 2];
                }
            }
        }
    };

    const bool late_wait = prefetch && xstatic;
    int row0 = gw * rows_per_batch + sub;                     // batch 0
    if (prefetch) load_pass(row0, 0);
    if (xstatic) build_table();
    if (dependent == 1 && !late_wait) grid_dependency_wait();
    if (!prefetch) load_pass(row0, 0);
    if (!xstatic) build_table();
    __syncthreads();

    const uint32_t lane_base = t0 + 4u * (uint32_t)lane;
    bool first = true;
    for (int b0 = gw * rows_per_batch; b0 < N; b0 += total_warps * rows_per_batch) {
        row0 = b0 + sub;
        float acc[U][4];
        #pragma unroll
        for (int u = 0; u < U; ++u)
            #pragma unroll
            for (int a = 0; a < 4; ++a) acc[u][a] = 0.0f;
        for (int p = 0; p < np; ++p) {
            if (!first || p > 0) load_pass(row0, p);
            const uint32_t lb = lane_base + (uint32_t)p * PASS_BYTES;
            // Rows innermost, so that consecutive adds belong to different rows.
            #pragma unroll
            for (int u = 0; u < U; ++u) bw_lookup_word<0>(v[u].x, lb, acc[u]);
            #pragma unroll
            for (int u = 0; u < U; ++u) bw_lookup_word<1>(v[u].y, lb, acc[u]);
            #pragma unroll
            for (int u = 0; u < U; ++u) bw_lookup_word<2>(v[u].z, lb, acc[u]);
            #pragma unroll
            for (int u = 0; u < U; ++u) bw_lookup_word<3>(v[u].w, lb, acc[u]);
        }
        #pragma unroll
        for (int u = 0; u < U; ++u) {
            float s = (acc[u][0] + acc[u][1]) + (acc[u][2] + acc[u][3]);
            if (lpr == 32) {                                  // a row spans the warp (K > 2048)
                #pragma unroll
                for (int off = 16; off >= 1; off >>= 1) s += __shfl_xor_sync(0xffffffffu, s, off);
            } else {
                for (int off = lpr >> 1; off >= 1; off >>= 1) s += __shfl_xor_sync(0xffffffffu, s, off);
            }
            acc[u][0] = s;
        }
        if (first && dependent == 1 && late_wait) grid_dependency_wait();
        first = false;
        if (li == 0) {
            #pragma unroll
            for (int u = 0; u < U; ++u) {
                const int r = row0 + u * rpi;
                if (r < N) y[r] = al[u] * acc[u][0];
            }
        }
    }
    if (dependent == 2) exit_after_previous_grid();
}

}  // namespace bnn
