// Integer-pipe rate probe: how many 32-bit population counts (POPC, the XU
// pipe), three-input logic ops (LOP3, the ALU pipe) and whole carry-save
// XOR-popcount words an SM retires per clock.  These are the denominators of
// the integer rooflines: "First Principles: Why Binary Ops Can Be
// Exponentially Faster", section "1. Arithmetic: MAC -> XNOR + popcount" --
// one 32-bit XOR + POPC replaces 32 binary multiply-accumulates, so a word
// rate times 32 is a binary MAC rate.
//
// Each mode runs register-only chains (no memory traffic inside the timed
// loop) on every SM, one 1024-thread CTA per SM, and times the loop with the
// SM clock (clock64).  Inline PTX keeps every operation opaque to the
// compiler, and each LOP3 mixes a different chain in as its third input so
// that no two dependent LOP3s can be merged into one.
//   mode 0: POPC only, 8 independent chains per thread.
//   mode 1: LOP3 only, 8 chains, each step reading its neighbour chain.
//   mode 2: the popcount GEMM's own inner step -- 8 XOR words compressed by
//           the 7:3 carry-save counter (4 POPC, 16 LOP3, 2 MAD, 1 IADD3) --
//           on 4 independent accumulators per thread.  Its rate in words per
//           clock is the roofline of that kernel's arithmetic.
#pragma once

#include "common.cuh"
#include "gemm_popc.cuh"   // full_add, mad_u32

namespace bnn {
namespace probe {
constexpr int THREADS = 1024;
constexpr int MAX_SMS = 1024;
constexpr int MODES = 3;
constexpr int CHAINS = 8;          // modes 0 and 1
constexpr int CSA_ACCS = 4;        // mode 2: independent accumulators per thread
// A dynamic shared-memory request larger than half an SM's shared memory
// keeps the grid at one CTA per SM.
constexpr int SMEM_BYTES = 160 * 1024;
}  // namespace probe

// Per-CTA elapsed SM clocks of the last probe launch, and a sink that keeps
// the chains' results alive.
__device__ unsigned long long g_probe_cycles[probe::MAX_SMS];
__device__ uint32_t g_probe_sink;

__device__ __forceinline__ uint32_t popc_op(uint32_t x) {
    uint32_t r;
    asm("popc.b32 %0, %1;" : "=r"(r) : "r"(x));
    return r;
}

template <int MODE>
__global__ void __launch_bounds__(probe::THREADS, 1) int_pipe_probe_kernel(int iters, uint32_t seed) {
    extern __shared__ uint8_t probe_smem[];
    (void)probe_smem;
    uint32_t v[probe::CHAINS];
    #pragma unroll
    for (int c = 0; c < probe::CHAINS; ++c) v[c] = (seed + 0x9E3779B9u * (threadIdx.x + 1)) ^ (0x85EBCA6Bu * c);
    __syncthreads();
    const unsigned long long t0 = clock64();
    if constexpr (MODE == 0) {
        #pragma unroll 1
        for (int it = 0; it < iters; ++it) {
            #pragma unroll
            for (int u = 0; u < 4; ++u) {
                #pragma unroll
                for (int c = 0; c < probe::CHAINS; ++c) v[c] = popc_op(v[c]) + 0u;
            }
        }
    } else if constexpr (MODE == 1) {
        #pragma unroll 1
        for (int it = 0; it < iters; ++it) {
            #pragma unroll
            for (int u = 0; u < 4; ++u) {
                uint32_t nv[probe::CHAINS];
                #pragma unroll
                for (int c = 0; c < probe::CHAINS; ++c) {
                    const uint32_t o = v[(c + 1 + u) % probe::CHAINS];
                    if ((c + u) & 1)
                        asm("lop3.b32 %0, %1, %2, %3, 0xe8;" : "=r"(nv[c]) : "r"(v[c]), "r"(o), "r"(seed));
                    else
                        asm("lop3.b32 %0, %1, %2, %3, 0x96;" : "=r"(nv[c]) : "r"(v[c]), "r"(o), "r"(seed));
                }
                #pragma unroll
                for (int c = 0; c < probe::CHAINS; ++c) v[c] = nv[c];
            }
        }
    } else {
        // v[0..7]: the 8 "activation" words of a row; each accumulator's own
        // running value supplies the "weight" word, so every step depends on
        // the previous one and nothing can be hoisted out of the loop.
        uint32_t acc[probe::CSA_ACCS];
        #pragma unroll
        for (int a = 0; a < probe::CSA_ACCS; ++a) acc[a] = seed + a;
        #pragma unroll 1
        for (int it = 0; it < iters; ++it) {
            #pragma unroll
            for (int a = 0; a < probe::CSA_ACCS; ++a) {
                uint32_t x[8];
                #pragma unroll
                for (int i = 0; i < 8; ++i)
                    asm("lop3.b32 %0, %1, %2, %3, 0x3c;" : "=r"(x[i]) : "r"(v[i]), "r"(acc[a]), "r"(0u));   // a ^ w
                acc[a] = popc8_csa_acc(x, acc[a]);
            }
        }
        #pragma unroll
        for (int a = 0; a < probe::CSA_ACCS; ++a) v[a] ^= acc[a];
    }
    __syncthreads();
    const unsigned long long t1 = clock64();          // the whole CTA is done (one SM clock counter)
    uint32_t s = 0;
    #pragma unroll
    for (int c = 0; c < probe::CHAINS; ++c) s ^= v[c];
    if (s == 0x12345678u) g_probe_sink = s;            // practically never taken; keeps the chains live
    if (threadIdx.x == 0 && blockIdx.x < probe::MAX_SMS) g_probe_cycles[blockIdx.x] = t1 - t0;
}

}  // namespace bnn
