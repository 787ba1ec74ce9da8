// A batch-1 chain of binary layers in one persistent launch: the decode step
// of a fully binary network, where each layer's input is the previous layer's
// re-binarised output.
//
// Each layer is the XNOR GEMV ("Extreme Quantization: Binary, Ternary & 1-bit
// LLMs", eq. (4) and (6): s = K - 2 popcount(w XOR x)); a hidden layer
// re-binarises through BatchNorm folded into an integer popcount threshold
// per channel (the THRESHOLD_PACK epilogue), the last layer returns int32 s
// and/or fp32 alpha_n * s (eq. (1)).  "First Principles: Why Binary Ops Can
// Be Exponentially Faster", "Bandwidth math": each layer streams its packed
// weights once, so the chain is bound by HBM as long as the hand-off between
// layers costs less than streaming one layer.
//
// Design (sm_100a, one launch for the whole chain):
//  * Cooperative launch, 2 blocks per SM, all resident.  Every block owns a
//    contiguous block of rows of every layer.
//  * A warp's rows of layer l+1 are loaded into registers (16-byte vectors,
//    lanes along the row) before the block waits for layer l's output.
//    (Asking L2 for later layers ahead of time, cp.async.bulk.prefetch.L2,
//    measured slower: the chain is bound by the per-layer hand-off, not by
//    the weight stream.)
//  * No grid barrier.  A hidden output word is a 64-bit slot
//    (tag << 40 | rows << 32 | bits): the warp that decides rows of a word
//    adds (rows decided << 32) | (their sign bits), one relaxed atomic add
//    per word after an acq_rel fence, and a block reading layer l's output
//    polls its words until every slot carries layer l's tag and counts all
//    of its rows (bounded by a timer; a warp-wide 8-byte load per 32 slots,
//    so each block sends one request per L2 line per round).  The wait for a
//    layer is then one L2 round trip after its last row is decided.
//  * Slots rotate through NBUF buffers.  Layer l resets the buffer layer l+2
//    will write to layer l+2's tag with no rows (the buffer was last read by
//    layer l-1, whose readers all finished before they contributed to layer
//    l-1's output, which this block has read); the resetting blocks are
//    active in layer l+1 too, so their next release orders the reset before
//    layer l+2.  The tag matters: a block with no rows in the layers before
//    one it owns rows of reaches that layer's wait early, possibly while the
//    buffer still holds the complete output of the layer NBUF earlier; the
//    tags differ, so it waits.  Layers 0 and 1 write buffers that start at
//    zero (tag 0); layer j >= 2 has tag j.  The last block to finish zeroes
//    every slot and the finish counter, so each launch starts from a zero
//    workspace.
//  * A timeout (one second per wait) sets the device error flag; the block
//    stops working but still reaches the finish counter, so the workspace is
//    zeroed for the next launch either way.
#pragma once

#include "common.cuh"

namespace bnn {
namespace chain {
constexpr int THREADS = 256;
constexpr int WARPS = THREADS / 32;
constexpr int SLOTS = 8;              // 16-byte weight vectors per lane per batch of rows
constexpr int MAX_LAYERS = 16;
constexpr int MAX_KW = 512;           // packed words per row: K <= 16384
constexpr int NBUF = 4;               // rotating hidden-output buffers of MAX_KW slots
constexpr int HEADER_WORDS = 16;      // workspace header (uint32): [0] = blocks finished
constexpr int WORKSPACE_WORDS = HEADER_WORDS + NBUF * MAX_KW * 2;
constexpr int POLL_GROUPS = MAX_KW / 32 / WARPS;   // 32-slot groups polled per warp
}  // namespace chain

struct ChainLayer {
    const uint32_t* W;       // packed [N, ldw]
    const int32_t* thr;      // hidden layers: popcount threshold per row
    const int8_t* mode;      // hidden layers: 0 -> bit = d > thr, 1 -> bit = d < thr
    const float* alpha;      // last layer: per-row scale (when fp32 output is asked for)
    int64_t ldw;
    int N, K, kw;            // outputs, inputs, packed words per row (multiple of 4)
    int rc;                  // rows per block
    int active;              // blocks that own rows: ceil(N / rc)
    int np;                  // 16-byte vectors per lane per row
    int lpr;                 // lanes per row (power of two)
    int lpr_log2;
    int zero_blocks;         // blocks that reset the buffer of layer l + 2 (0: none)
    int zero_words;          // slots layer l + 2 writes
    int zero_per;            // slots each resetting block clears
};

struct ChainArgs {
    ChainLayer layer[chain::MAX_LAYERS];
    const void* x;                 // real input of layer 0, [K0]
    int32_t* y_i32;                // last layer outputs (either may be null)
    float* y_f32;
    uint32_t* acts;                // optional: hidden outputs, packed rows [L - 1, ld_acts]
    int64_t ld_acts;
    unsigned long long* slots;     // [NBUF][MAX_KW]
    unsigned int* finished;
    int L;
    int x_vec;                     // x is 16-byte aligned
};

// Tag of the slots layer j writes (see the design notes above).
__device__ __forceinline__ uint32_t chain_tag(int j) { return j < 2 ? 0u : (uint32_t)j; }

// This warp's rows of a layer: [lo, hi), in row groups of rpi rows (one row
// per lpr lanes), SLOTS / NP row groups per batch.
struct WarpRows {
    int lo, hi, rpi, li, sub;
};

__device__ __forceinline__ WarpRows warp_rows(const ChainLayer& ly, int blk, int warp, int lane) {
    using namespace chain;
    WarpRows w;
    const int b_lo = blk * ly.rc;
    const int b_hi = min(ly.N, b_lo + ly.rc);
    const int rw = (ly.rc + WARPS - 1) / WARPS;
    w.lo = min(b_hi, b_lo + warp * rw);
    w.hi = min(b_hi, w.lo + rw);
    w.rpi = 32 >> ly.lpr_log2;
    w.li = lane & (ly.lpr - 1);
    w.sub = lane >> ly.lpr_log2;
    return w;
}

// Predicated read-only loads into registers the caller has zeroed: nothing
// consumes the destination until the data is used, so a warp issues all of
// its loads back to back and only waits where it computes.
__device__ __forceinline__ void ldg_v4_if(uint4& v, const void* p, bool pred) {
    asm volatile(
        "{\n\t.reg .pred q;\n\tsetp.ne.b32 q, %5, 0;\n\t"
        "@q ld.global.nc.L1::no_allocate.v4.u32 {%0, %1, %2, %3}, [%4];\n\t}"
        : "+r"(v.x), "+r"(v.y), "+r"(v.z), "+r"(v.w)
        : "l"(p), "r"((int)pred));
}
__device__ __forceinline__ void ldg_b32_if(uint32_t& v, const void* p, bool pred) {
    asm volatile("{\n\t.reg .pred q;\n\tsetp.ne.b32 q, %2, 0;\n\t@q ld.global.nc.b32 %0, [%1];\n\t}"
                 : "+r"(v) : "l"(p), "r"((int)pred));
}
__device__ __forceinline__ void ldg_s8_if(uint32_t& v, const void* p, bool pred) {
    asm volatile("{\n\t.reg .pred q;\n\tsetp.ne.b32 q, %2, 0;\n\t@q ld.global.nc.s8 %0, [%1];\n\t}"
                 : "+r"(v) : "l"(p), "r"((int)pred));
}

// Loads batch `b` of this warp's rows: the weight vectors and, for the lane
// that finishes a row (li == 0), the row's epilogue parameters (hidden
// layers: threshold in e0, mode in e1; last layer: alpha's bits in e0).
template <int NP>
__device__ __forceinline__ void chain_load(const ChainLayer& ly, const WarpRows& w, int b, bool last,
                                           uint4 (&v)[chain::SLOTS], uint32_t (&e0)[chain::SLOTS],
                                           uint32_t (&e1)[chain::SLOTS]) {
    constexpr int GB = chain::SLOTS / NP;
    const int nch = ly.kw / 4;
    const int r0 = w.lo + b * GB * w.rpi + w.sub;
    #pragma unroll
    for (int g = 0; g < GB; ++g) {
        const int r = r0 + g * w.rpi;
        const bool ok = r < w.hi;
        #pragma unroll
        for (int p = 0; p < NP; ++p) {
            const int c = w.li + ly.lpr * p;
            v[g * NP + p] = make_uint4(0u, 0u, 0u, 0u);
            ldg_v4_if(v[g * NP + p], ly.W + (int64_t)r * ly.ldw + 4 * c, ok && c < nch);
        }
        e0[g] = 0u;
        e1[g] = 0u;
        const bool mine = ok && w.li == 0;
        if (last) {
            ldg_b32_if(e0[g], ly.alpha + r, mine && ly.alpha != nullptr);
        } else {
            ldg_b32_if(e0[g], ly.thr + r, mine);
            ldg_s8_if(e1[g], ly.mode + r, mine);
        }
    }
}

// One batch: popcounts of the rows against x (xs, shared memory), then the
// epilogue.  Hidden layers add their decisions to the output slots.
template <int NP>
__device__ __forceinline__ void chain_batch(const ChainLayer& ly, const WarpRows& w, int b, bool last,
                                            const uint32_t* xs, const uint4 (&v)[chain::SLOTS],
                                            const uint32_t (&e0)[chain::SLOTS], const uint32_t (&e1)[chain::SLOTS],
                                            unsigned long long* out_slots,
                                            int32_t* y_i32, float* y_f32, int lane) {
    constexpr int GB = chain::SLOTS / NP;
    const int nch = ly.kw / 4;
    uint4 xq[NP];
    #pragma unroll
    for (int p = 0; p < NP; ++p) {
        const int c = w.li + ly.lpr * p;
        xq[p] = c < nch ? *reinterpret_cast<const uint4*>(xs + 4 * c) : make_uint4(0u, 0u, 0u, 0u);
    }
    uint32_t d[GB];
    #pragma unroll
    for (int g = 0; g < GB; ++g) {
        uint32_t acc = 0;
        #pragma unroll
        for (int p = 0; p < NP; ++p) acc += popc_xor4(v[g * NP + p], xq[p]);
        if (ly.lpr == 32) {
            acc = __reduce_add_sync(0xffffffffu, acc);
        } else {
            for (int off = ly.lpr >> 1; off >= 1; off >>= 1) acc += __shfl_xor_sync(0xffffffffu, acc, off);
        }
        d[g] = acc;
    }
    const int rb0 = w.lo + b * GB * w.rpi;                 // first row of the batch
    const int r0 = rb0 + w.sub;
    if (last) {
        #pragma unroll
        for (int g = 0; g < GB; ++g) {
            const int r = r0 + g * w.rpi;
            if (w.li == 0 && r < w.hi) {
                const int32_t s = ly.K - 2 * (int32_t)d[g];
                if (y_i32 != nullptr) y_i32[r] = s;
                if (y_f32 != nullptr) y_f32[r] = __uint_as_float(e0[g]) * (float)s;
            }
        }
        return;
    }
    const int rb1 = min(w.hi, rb0 + GB * w.rpi);
    if (rb1 <= rb0) return;                                // warp-uniform
    for (int wd = rb0 >> 5; wd <= (rb1 - 1) >> 5; ++wd) {  // the slots this batch's rows fall in
        uint32_t bits = 0, cnt = 0;
        #pragma unroll
        for (int g = 0; g < GB; ++g) {
            const int r = r0 + g * w.rpi;
            if (w.li == 0 && r < w.hi && (r >> 5) == wd) {
                const int thr = (int)e0[g];
                const bool bit = e1[g] != 0u ? ((int)d[g] < thr) : ((int)d[g] > thr);
                bits |= (bit ? 1u : 0u) << (r & 31);
                cnt += 1;
            }
        }
        bits = __reduce_or_sync(0xffffffffu, bits);
        cnt = __reduce_add_sync(0xffffffffu, cnt);
        if (lane == 0 && cnt != 0) {
            const unsigned long long add = ((unsigned long long)cnt << 32) | bits;
            asm volatile("red.relaxed.gpu.global.add.u64 [%0], %1;" ::"l"(out_slots + wd), "l"(add) : "memory");
        }
    }
}

// All of this warp's rows of a layer; batch 0 was loaded before the wait.
template <int NP>
__device__ __forceinline__ void chain_rows(const ChainLayer& ly, const WarpRows& w, bool last, const uint32_t* xs,
                                           uint4 (&v)[chain::SLOTS], uint32_t (&e0)[chain::SLOTS],
                                           uint32_t (&e1)[chain::SLOTS], unsigned long long* out_slots,
                                           int32_t* y_i32, float* y_f32, int lane) {
    constexpr int GB = chain::SLOTS / NP;
    if (w.hi <= w.lo) return;
    const int groups = (w.hi - w.lo + w.rpi - 1) >> (5 - ly.lpr_log2);   // rpi = 2^(5 - lpr_log2)
    const int batches = (groups + GB - 1) / GB;
    for (int b = 0; b < batches; ++b) {
        if (b > 0) chain_load<NP>(ly, w, b, last, v, e0, e1);
        chain_batch<NP>(ly, w, b, last, xs, v, e0, e1, out_slots, y_i32, y_f32, lane);
    }
}

__device__ __forceinline__ void chain_load_any(const ChainLayer& ly, const WarpRows& w, bool last,
                                               uint4 (&v)[chain::SLOTS], uint32_t (&e0)[chain::SLOTS],
                                               uint32_t (&e1)[chain::SLOTS]) {
    if (w.hi <= w.lo) return;
    switch (ly.np) {
        case 1: chain_load<1>(ly, w, 0, last, v, e0, e1); break;
        case 2: chain_load<2>(ly, w, 0, last, v, e0, e1); break;
        case 3: chain_load<3>(ly, w, 0, last, v, e0, e1); break;
        default: chain_load<4>(ly, w, 0, last, v, e0, e1); break;
    }
}

// Waits (bounded) until every slot of the input buffer carries the producing
// layer's tag and all of its rows, then writes the K input bits to xs (zero
// up to kw words).  Warp w polls the 32-slot groups w, w + WARPS, ...; a
// group is re-read until complete.  Returns false on a timeout.  Ends with
// an acq_rel fence: the acquire side of the slot reads and the release side
// of this layer's adds.
__device__ __forceinline__ bool chain_poll(const unsigned long long* in_slots, uint32_t tag, int K, int kw,
                                           uint32_t* xs, int warp, int lane) {
    using namespace chain;
    const int nw = (K + 31) / 32;
    bool ok = true;
    unsigned long long t0 = 0;
    #pragma unroll
    for (int j = 0; j < POLL_GROUPS; ++j) {
        const int wd = (warp + WARPS * j) * 32 + lane;
        if ((warp + WARPS * j) * 32 >= kw) break;             // warp-uniform
        uint32_t bits = 0;
        if (ok) {
            const uint32_t expect = wd < nw ? (tag << 8) | (uint32_t)min(32, K - 32 * wd) : 0u;
            for (int it = 0;; ++it) {
                unsigned long long val = 0;
                if (wd < nw)
                    asm volatile("ld.relaxed.gpu.global.u64 %0, [%1];" : "=l"(val) : "l"(in_slots + wd) : "memory");
                const bool done = (uint32_t)(val >> 32) == expect;
                if (__all_sync(0xffffffffu, done)) {
                    bits = (uint32_t)val;
                    break;
                }
                if ((it & 15) == 15) {
                    // lane 0's clock decides, so the warp leaves together
                    const unsigned long long t = __shfl_sync(0xffffffffu, globaltimer_ns(), 0);
                    if (t0 == 0) {
                        t0 = t;
                    } else if (t - t0 > kWaitTimeoutNs) {
                        ok = false;
                        break;
                    }
                }
            }
        }
        if (wd < kw) xs[wd] = bits;
    }
    asm volatile("fence.acq_rel.gpu;" ::: "memory");
    return ok;
}

// The real input of layer 0 packed by sign into xs (bit 1 = x < 0), zero up
// to kw words; the trip count is block-uniform so full-warp shuffles stay
// converged.
template <typename XT>
__device__ __forceinline__ void chain_pack_x(const XT* __restrict__ x, int K, int kw, bool vec, uint32_t* xs) {
    using namespace chain;
    constexpr int E = 16 / (int)sizeof(XT);
    constexpr int G = 32 / E;
    const int nvec = kw * G;
    const int nfull = vec ? K / E : 0;
    for (int c0 = 0; c0 < nvec; c0 += THREADS) {
        const int c = c0 + (int)threadIdx.x;
        uint32_t b = 0;
        if (c < nfull) {
            const uint4 q = *reinterpret_cast<const uint4*>(x + E * c);
            const XT* e = reinterpret_cast<const XT*>(&q);
            #pragma unroll
            for (int i = 0; i < E; ++i) b |= neg_bit(to_float(e[i])) << i;
        } else if (c < nvec) {
            for (int i = 0; i < E; ++i) {
                const int k = E * c + i;
                if (k < K) b |= neg_bit(to_float(x[k])) << i;
            }
        }
        b <<= E * (c & (G - 1));
        #pragma unroll
        for (int off = 1; off < G; off <<= 1) b |= __shfl_xor_sync(0xffffffffu, b, off);
        if ((c & (G - 1)) == 0 && c < nvec) xs[c / G] = b;
    }
}

template <typename XT>
__global__ void __launch_bounds__(chain::THREADS, 2)
xnor_gemv_chain_kernel(const __grid_constant__ ChainArgs a) {
    using namespace chain;
    __shared__ __align__(16) uint32_t xs[MAX_KW];
    __shared__ __align__(16) ChainLayer layers[MAX_LAYERS];
    __shared__ int s_last;
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int blk = blockIdx.x;

    // The layer table is read at every layer boundary with a runtime index;
    // from the parameter space that is a chain of dependent constant-cache
    // misses, so it is copied to shared memory once.
    {
        static_assert(sizeof(ChainLayer) % 4 == 0, "layer table copied in words");
        const uint32_t* src = reinterpret_cast<const uint32_t*>(&a.layer[0]);
        uint32_t* dst = reinterpret_cast<uint32_t*>(layers);
        const int n = a.L * (int)(sizeof(ChainLayer) / 4);
        for (int i = threadIdx.x; i < n; i += THREADS) dst[i] = src[i];
    }
    __syncthreads();

    uint4 v[SLOTS];
    uint32_t e0[SLOTS], e1[SLOTS];
    // The current and the next layer's parameters live in registers: through
    // a reference the compiler would re-read them after every asm statement
    // that clobbers memory.
    ChainLayer nx = layers[0];
    WarpRows w = warp_rows(nx, blk, warp, lane);
    if (blk < nx.active) {
        chain_load_any(nx, w, a.L == 1, v, e0, e1);
        chain_pack_x(static_cast<const XT*>(a.x), nx.K, nx.kw, a.x_vec != 0, xs);
    }
    __syncthreads();

    for (int l = 0; l < a.L; ++l) {
        const ChainLayer ly = nx;
        const bool last = l == a.L - 1;
        const bool act = blk < ly.active;
        unsigned long long* out_slots = a.slots + (size_t)(l % NBUF) * MAX_KW;
        if (l > 0) {
            // every warp is done with layer l - 1 (xs reads, adds, zeroes)
            __syncthreads();
            bool mine = true;
            if (act) {
                mine = chain_poll(a.slots + (size_t)((l - 1) % NBUF) * MAX_KW, chain_tag(l - 1), ly.K, ly.kw, xs,
                                  warp, lane);
            }
            if (__syncthreads_or(mine ? 0 : 1)) {
                if (threadIdx.x == 0) flag_device_error(BNN_ERR_DEVICE_TIMEOUT);
                break;
            }
            if (blk == 0 && a.acts != nullptr) {
                for (int i = threadIdx.x; i < ly.kw; i += THREADS) a.acts[(int64_t)(l - 1) * a.ld_acts + i] = xs[i];
            }
        }
        if (act) {
            switch (ly.np) {
                case 1: chain_rows<1>(ly, w, last, xs, v, e0, e1, out_slots, a.y_i32, a.y_f32, lane); break;
                case 2: chain_rows<2>(ly, w, last, xs, v, e0, e1, out_slots, a.y_i32, a.y_f32, lane); break;
                case 3: chain_rows<3>(ly, w, last, xs, v, e0, e1, out_slots, a.y_i32, a.y_f32, lane); break;
                default: chain_rows<4>(ly, w, last, xs, v, e0, e1, out_slots, a.y_i32, a.y_f32, lane); break;
            }
        }
        // reset the buffer layer l + 2 writes (its slots were last read by layer l - 1)
        if (blk < ly.zero_blocks) {
            unsigned long long* z = a.slots + (size_t)((l + 2) % NBUF) * MAX_KW;
            const unsigned long long base = (unsigned long long)chain_tag(l + 2) << 40;
            const int z1 = min(ly.zero_words, (blk + 1) * ly.zero_per);
            for (int i = blk * ly.zero_per + (int)threadIdx.x; i < z1; i += THREADS) z[i] = base;
        }
        if (!last) {
            nx = layers[l + 1];
            w = warp_rows(nx, blk, warp, lane);
            if (blk < nx.active) chain_load_any(nx, w, l + 1 == a.L - 1, v, e0, e1);
        }
    }

    // The last block to finish leaves a zero workspace for the next launch.
    __syncthreads();
    if (threadIdx.x == 0) {
        unsigned int prev;
        asm volatile("atom.acq_rel.gpu.global.add.u32 %0, [%1], 1;" : "=r"(prev) : "l"(a.finished) : "memory");
        s_last = prev == gridDim.x - 1 ? 1 : 0;
    }
    __syncthreads();
    if (s_last) {
        for (int i = threadIdx.x; i < NBUF * MAX_KW; i += THREADS) a.slots[i] = 0ull;
        __syncthreads();
        if (threadIdx.x == 0) *a.finished = 0u;
    }
}

}  // namespace bnn
