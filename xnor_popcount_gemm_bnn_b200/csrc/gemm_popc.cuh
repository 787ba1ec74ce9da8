// Packed binary GEMM on the integer pipes: d[m, n] = sum_w popcount(A[m, w]
// XOR W[n, w]), s = K - 2 d ("Extreme Quantization: Binary, Ternary & 1-bit
// LLMs", XNOR-Net eq. (6); "First Principles: Why Binary Ops Can Be
// Exponentially Faster", section 1), with a fused epilogue: int32 s, alpha*s
// (eq. (1)), gamma*(alpha*s)+beta, or a popcount threshold re-packed into
// sign bits for the next layer (folded BatchNorm).
//
// Design (sm_100a):
//  * CTA tile BM x BN outputs (BM = 128, BN = 16 * TN), K staged 32 words
//    (1024 binary elements) at a time.  One producer warp issues TMA tile
//    loads (no multicast) into a 4-stage ring of 128B-swizzled shared-memory
//    tiles; completion is tracked with mbarriers (full: TMA bytes landed;
//    empty: all 8 compute warps are done with the stage).  Every wait is
//    bounded (about 1 s) and reports BNN_ERR_DEVICE_TIMEOUT instead of hanging.
//  * 8 compute warps; thread (tx, ty) of a 16 x 16 grid owns rows ty + 16 i
//    (i < 8) and columns tx + 16 j (j < TN).  The 128B swizzle makes the 8
//    rows read by a quarter warp fall on 8 distinct 16-byte bank groups.
//  * Population count runs on the XU pipe at 16 per clock per SM, logic ops
//    on the ALU pipe at 64 per clock.  With CSA (carry-save) the thread takes
//    8 XOR words per (row, column) at a time and compresses 7 of them with a
//    7:3 counter built from four full adders (sum = a^b^c, carry = majority:
//    one LOP3 each), so 8 words cost 4 POPC instead of 8:
//        popc(x0..x7) = popc(s) + popc(x7) + 2 popc(t) + 4 popc(u).
//    That moves work from the saturated XU pipe onto the ALU pipe.
//  * Zero-filled out-of-range TMA boxes make ragged M, N and K (pad words)
//    contribute nothing to d (XOR of zeros is zero; so are its adder sums).
#pragma once

#include "common.cuh"

namespace bnn {
namespace gemm {
constexpr int BM = 128;
constexpr int BKW = 32;                      // words per K stage (128 bytes per row)
constexpr int STAGES = 4;
constexpr int COMPUTE_WARPS = 8;
constexpr int THREADS = (COMPUTE_WARPS + 1) * 32;
constexpr int A_TILE_BYTES = BM * BKW * 4;   // 16 KiB

// Product configuration: 8 x 4 register tile with carry-save compression.
constexpr int TN = 4;
constexpr bool CSA = true;
constexpr int BN = 16 * TN;
constexpr int W_TILE_BYTES = BN * BKW * 4;
constexpr int STAGE_BYTES = A_TILE_BYTES + W_TILE_BYTES;
constexpr int SMEM_BYTES = STAGES * STAGE_BYTES + 2 * STAGES * 8 + 1024;
}  // namespace gemm

struct GemmEpilogue {
    int32_t* c_i32;           // int32 s, or null
    int64_t ldc;
    float* c_f32;             // alpha*s (or gamma*(alpha*s)+beta when gamma != null), or null
    int64_t ldf;
    const float* alpha;
    const float* gamma;
    const float* beta;
    uint32_t* c_bits;         // THRESHOLD_PACK output, or null
    int64_t ldb;              // words
    int64_t bits_words;       // packed words per output row (bnn_packed_ld_words(N))
    const int32_t* thresh;
    const int8_t* thresh_mode;
};

// One full adder on 32 bit-slices: sum = a ^ b ^ c (LOP3 truth table 0x96),
// carry = majority(a, b, c) (0xE8).  Written as one LOP3 each so that the
// compiler does not share a ^ b between them (which costs a third LOP3).
__device__ __forceinline__ void full_add(uint32_t a, uint32_t b, uint32_t c, uint32_t& sum, uint32_t& carry) {
    asm("lop3.b32 %0, %1, %2, %3, 0x96;" : "=r"(sum) : "r"(a), "r"(b), "r"(c));
    asm("lop3.b32 %0, %1, %2, %3, 0xe8;" : "=r"(carry) : "r"(a), "r"(b), "r"(c));
}

// acc + x * k on the FMA pipe (integer multiply-add), leaving the ALU pipe to
// the logic ops.
__device__ __forceinline__ uint32_t mad_u32(uint32_t x, uint32_t k, uint32_t acc) {
    uint32_t r;
    asm("mad.lo.u32 %0, %1, %2, %3;" : "=r"(r) : "r"(x), "r"(k), "r"(acc));
    return r;
}

// acc + popcount(x0) + ... + popcount(x7) with four POPC: a 7:3 counter on
// x0..x6 (outputs of weight 1, 2, 4) plus x7.
__device__ __forceinline__ uint32_t popc8_csa_acc(const uint32_t (&x)[8], uint32_t acc) {
    uint32_t s1, c1, s2, c2, s3, c3, s4, c4;
    full_add(x[0], x[1], x[2], s1, c1);
    full_add(x[3], x[4], x[5], s2, c2);
    full_add(s1, s2, x[6], s3, c3);      // s3: weight 1, c3: weight 2
    full_add(c1, c2, c3, s4, c4);        // s4: weight 2, c4: weight 4
    acc = mad_u32(__popc(s4), 2u, acc);
    acc = mad_u32(__popc(c4), 4u, acc);
    return acc + __popc(s3) + __popc(x[7]);
}

__device__ __forceinline__ uint32_t popc8_csa(const uint32_t (&x)[8]) { return popc8_csa_acc(x, 0u); }

template <int TN_, bool CSA_>
__global__ void __launch_bounds__(gemm::THREADS, 1)
xnor_gemm_popc_kernel(const __grid_constant__ CUtensorMap tmA, const __grid_constant__ CUtensorMap tmW,
                      int M, int N, int K, int kw, int tiles_n, GemmEpilogue ep) {
    using namespace gemm;
    constexpr int BN_ = 16 * TN_;
    constexpr int W_BYTES = BN_ * BKW * 4;
    constexpr int STAGE = A_TILE_BYTES + W_BYTES;
    extern __shared__ uint8_t smem_raw[];
    // 1024-byte aligned base, derived by offset from the __shared__ array so
    // that the compiler keeps every access in the shared address space.
    uint8_t* smem = smem_raw + ((1024u - (smem_u32(smem_raw) & 1023u)) & 1023u);
    uint64_t* full = reinterpret_cast<uint64_t*>(smem + STAGES * STAGE);
    uint64_t* empty = full + STAGES;

    const int warp = threadIdx.x >> 5;
    const int lane = threadIdx.x & 31;
    const int tile_m = blockIdx.x / tiles_n;
    const int tile_n = blockIdx.x % tiles_n;
    const int m0 = tile_m * BM;
    const int n0 = tile_n * BN_;
    const int nk = (kw + BKW - 1) / BKW;

    if (threadIdx.x == 0) {
        prefetch_tensormap(&tmA);
        prefetch_tensormap(&tmW);
        #pragma unroll
        for (int s = 0; s < STAGES; ++s) {
            mbar_init(&full[s], 1);
            mbar_init(&empty[s], COMPUTE_WARPS);
        }
        fence_mbarrier_init();
    }
    __syncthreads();

    if (warp == COMPUTE_WARPS) {
        // ---------------- producer warp ----------------
        if (lane == 0) {
            int issued = 0;
            for (int kt = 0; kt < nk; ++kt) {
                const int s = kt % STAGES;
                const uint32_t ph = (kt / STAGES) & 1;
                if (kt >= STAGES && !mbar_wait_bounded(&empty[s], ph ^ 1)) break;
                uint8_t* sa = smem + s * STAGE;
                mbar_arrive_expect_tx(&full[s], STAGE);
                tma_load_2d(sa, &tmA, kt * BKW, m0, &full[s]);
                tma_load_2d(sa + A_TILE_BYTES, &tmW, kt * BKW, n0, &full[s]);
                ++issued;
            }
            // Do not let the CTA retire while copies are still landing.
            for (int kt = max(0, issued - STAGES); kt < issued; ++kt)
                if (!mbar_wait_bounded(&full[kt % STAGES], (kt / STAGES) & 1)) break;
        }
        return;
    }

    // ---------------- compute warps ----------------
    const int t = threadIdx.x;
    const int tx = t & 15;
    const int ty = t >> 4;
    const int swa = ty & 7;   // (ty + 16 i) & 7
    const int swb = tx & 7;   // (tx + 16 j) & 7
    uint32_t acc[8][TN_];
    #pragma unroll
    for (int i = 0; i < 8; ++i)
        #pragma unroll
        for (int j = 0; j < TN_; ++j) acc[i][j] = 0u;

    for (int kt = 0; kt < nk; ++kt) {
        const int s = kt % STAGES;
        // Warp-uniform decision, so that no lane leaves while others reach a ballot.
        if (!__all_sync(0xffffffffu, mbar_wait_bounded(&full[s], (kt / STAGES) & 1))) return;
        const uint8_t* As = smem + s * STAGE;
        const uint8_t* Ws = As + A_TILE_BYTES;
        if constexpr (CSA_) {
            #pragma unroll 1
            for (int c = 0; c < BKW / 4; c += 2) {        // two 16-byte chunks = 8 words
                uint32_t a[8][8], b[TN_][8];
                #pragma unroll
                for (int i = 0; i < 8; ++i) {
                    const uint8_t* row = As + (ty + 16 * i) * 128;
                    const uint4 q0 = *reinterpret_cast<const uint4*>(row + ((c ^ swa) << 4));
                    const uint4 q1 = *reinterpret_cast<const uint4*>(row + (((c + 1) ^ swa) << 4));
                    a[i][0] = q0.x; a[i][1] = q0.y; a[i][2] = q0.z; a[i][3] = q0.w;
                    a[i][4] = q1.x; a[i][5] = q1.y; a[i][6] = q1.z; a[i][7] = q1.w;
                }
                #pragma unroll
                for (int j = 0; j < TN_; ++j) {
                    const uint8_t* row = Ws + (tx + 16 * j) * 128;
                    const uint4 q0 = *reinterpret_cast<const uint4*>(row + ((c ^ swb) << 4));
                    const uint4 q1 = *reinterpret_cast<const uint4*>(row + (((c + 1) ^ swb) << 4));
                    b[j][0] = q0.x; b[j][1] = q0.y; b[j][2] = q0.z; b[j][3] = q0.w;
                    b[j][4] = q1.x; b[j][5] = q1.y; b[j][6] = q1.z; b[j][7] = q1.w;
                }
                #pragma unroll
                for (int i = 0; i < 8; ++i)
                    #pragma unroll
                    for (int j = 0; j < TN_; ++j) {
                        uint32_t x[8];
                        #pragma unroll
                        for (int k = 0; k < 8; ++k) x[k] = a[i][k] ^ b[j][k];
                        acc[i][j] = popc8_csa_acc(x, acc[i][j]);
                    }
            }
        } else {
            #pragma unroll 2
            for (int c = 0; c < BKW / 4; ++c) {
                uint4 a[8], b[TN_];
                #pragma unroll
                for (int i = 0; i < 8; ++i)
                    a[i] = *reinterpret_cast<const uint4*>(As + (ty + 16 * i) * 128 + ((c ^ swa) << 4));
                #pragma unroll
                for (int j = 0; j < TN_; ++j)
                    b[j] = *reinterpret_cast<const uint4*>(Ws + (tx + 16 * j) * 128 + ((c ^ swb) << 4));
                #pragma unroll
                for (int i = 0; i < 8; ++i)
                    #pragma unroll
                    for (int j = 0; j < TN_; ++j) acc[i][j] += popc_xor4(a[i], b[j]);
            }
        }
        // The stage's words were read through the generic proxy; the
        // producer refills it with TMA (async proxy) once `empty` completes.
        // The proxy fence orders those reads before that write.
        fence_proxy_async_shared();
        __syncwarp();
        if (lane == 0) mbar_arrive(&empty[s]);
    }

    // ---------------- epilogue ----------------
    if (ep.c_i32 != nullptr || ep.c_f32 != nullptr) {
        float al[TN_], ga[TN_], be[TN_];
        #pragma unroll
        for (int j = 0; j < TN_; ++j) {
            const int n = n0 + tx + 16 * j;
            const bool in = n < N;
            al[j] = (ep.alpha != nullptr && in) ? ep.alpha[n] : 0.0f;
            ga[j] = (ep.gamma != nullptr && in) ? ep.gamma[n] : 0.0f;
            be[j] = (ep.beta != nullptr && in) ? ep.beta[n] : 0.0f;
        }
        #pragma unroll
        for (int i = 0; i < 8; ++i) {
            const int m = m0 + ty + 16 * i;
            if (m >= M) continue;
            #pragma unroll
            for (int j = 0; j < TN_; ++j) {
                const int n = n0 + tx + 16 * j;
                if (n >= N) continue;
                const int32_t sv = K - 2 * (int32_t)acc[i][j];
                if (ep.c_i32 != nullptr) ep.c_i32[(int64_t)m * ep.ldc + n] = sv;
                if (ep.c_f32 != nullptr) {
                    float y = al[j] * (float)sv;
                    if (ep.gamma != nullptr) y = fmaf(ga[j], y, be[j]);
                    ep.c_f32[(int64_t)m * ep.ldf + n] = y;
                }
            }
        }
    }
    if (ep.c_bits != nullptr) {
        int32_t th[TN_];
        int8_t md[TN_];
        #pragma unroll
        for (int j = 0; j < TN_; ++j) {
            const int n = n0 + tx + 16 * j;
            th[j] = (n < N) ? ep.thresh[n] : 0;
            md[j] = (n < N) ? ep.thresh_mode[n] : (int8_t)-1;   // -1: column past N, bit 0
        }
        #pragma unroll
        for (int i = 0; i < 8; ++i) {
            const int m_even = m0 + 2 * warp + 16 * i;   // lanes 0..15 hold row ty = 2*warp
            #pragma unroll
            for (int q = 0; q < TN_ / 2; ++q) {           // word q of the tile's columns
                const int j0 = 2 * q, j1 = 2 * q + 1;
                const int32_t d0 = (int32_t)acc[i][j0], d1 = (int32_t)acc[i][j1];
                const bool bit0 = md[j0] == 0 ? (d0 > th[j0]) : (md[j0] == 1 ? (d0 < th[j0]) : false);
                const bool bit1 = md[j1] == 0 ? (d1 > th[j1]) : (md[j1] == 1 ? (d1 < th[j1]) : false);
                const uint32_t b0 = __ballot_sync(0xffffffffu, bit0);
                const uint32_t b1 = __ballot_sync(0xffffffffu, bit1);
                const int64_t word = n0 / 32 + q;
                if (word < ep.bits_words) {
                    if (lane == 0 && m_even < M)
                        ep.c_bits[(int64_t)m_even * ep.ldb + word] = (b0 & 0xffffu) | (b1 << 16);
                    if (lane == 16 && m_even + 1 < M)
                        ep.c_bits[(int64_t)(m_even + 1) * ep.ldb + word] = (b0 >> 16) | (b1 & 0xffff0000u);
                }
            }
        }
        // The last column tile also zeroes the pad words that no tile covers.
        if (tile_n == tiles_n - 1) {
            const int64_t first_pad = (int64_t)(n0 + BN_) / 32;
            for (int64_t w = first_pad + tx; w < ep.bits_words; w += 16) {
                #pragma unroll
                for (int i = 0; i < 8; ++i) {
                    const int m = m0 + ty + 16 * i;
                    if (m < M) ep.c_bits[(int64_t)m * ep.ldb + w] = 0u;
                }
            }
        }
    }
}

}  // namespace bnn
