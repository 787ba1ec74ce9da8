// Packed binary GEMM on the 5th-generation tensor cores (tcgen05, kind::i8).
//
// Same product as gemm_popc.cuh -- s[m, n] = sum_k a_mk * w_nk over +1/-1
// values ("Extreme Quantization: Binary, Ternary & 1-bit LLMs", eq. (1), (4)
// and (6)) -- computed by expanding the packed sign bits to signed bytes
// (bit 0 -> +1 = 0x01, bit 1 -> -1 = 0xFF) in shared memory and multiplying
// them with tcgen05.mma kind::i8 into int32 accumulators in tensor memory.
// Every product is +1 or -1 and the accumulation is exact in int32, so the
// result is bit-identical to K - 2 * popcount(A XOR W).  Pad positions (bits
// past K inside the packed rows, and zero-filled words past the row end) are
// 0 bits in both operands, i.e. (+1)(+1) = +1 each; the epilogue subtracts
// their count, (K rounded up to a whole stage) - K.
//
// Design (sm_100a, one persistent CTA per SM, 18 warps):
//  * warp 0   : TMA producer.  Packed tiles (128 A rows x 4 words, 256 W rows
//               x 4 words = 128 binary elements of K) into an 8-stage ring.
//  * warps 2-13: unpack, one thread per packed row of the stage (128 A rows,
//               256 W rows).  Each packed word becomes 32 signed bytes in the
//               K-major 128B-swizzled layout the tensor core reads (chunk c of
//               row r at (c ^ (r & 7)) * 16); four ops per 4 bytes (PRMT picks
//               a nibble, IMAD spreads its bits into bytes, LOP3 masks, IMAD
//               maps {0,1} to {+1,-1}).  fence.proxy.async, then an mbarrier
//               arrive hands the stage to the MMA warp.
//  * warp 1   : allocates 512 TMEM columns (two 128 x 256 int32 accumulators);
//               one thread issues 4 tcgen05.mma (M=128, N=256, K=32) per stage
//               and commits them to the stage's "empty" barrier, and to the
//               accumulator's "full" barrier after the last stage of a tile.
//  * warps 14-17: epilogue.  Warp q reads TMEM lanes 32q..32q+31 (one output
//               row per thread) 32 columns at a time with tcgen05.ld, releases
//               the accumulator, and writes int32 / alpha*s / affine outputs or
//               the folded-BatchNorm sign bits (32 columns = one packed word,
//               all in one thread).  Double buffering lets the epilogue of tile
//               i overlap the MMAs of tile i+1.
//  * Every mbarrier wait is bounded (about 1 s): on time-out the CTA records
//    BNN_ERR_DEVICE_TIMEOUT, the other roles stop at their next wait, the MMA
//    thread waits (bounded) for its last MMAs, and TMEM is freed before exit.
#pragma once

#include "common.cuh"
#include "gemm_popc.cuh"   // GemmEpilogue

namespace bnn {
namespace tc {
constexpr int BM = 128;                    // tile rows  = TMEM lanes = UMMA M
constexpr int BN = 256;                    // tile cols  = UMMA N
constexpr int BKE = 128;                   // elements of K per stage (4 packed words)
constexpr int BKW = BKE / 32;
constexpr int UMMA_K = 32;                 // int8 K per tcgen05.mma
constexpr int PSTAGES = 8;                 // packed ring (binary and bases modes)
constexpr int USTAGES = 3;                 // unpacked (int8) ring
constexpr int P_A_BYTES = BM * BKW * 4;    // 2 KiB
constexpr int P_B_BYTES = BN * BKW * 4;    // 4 KiB
constexpr int P_STAGE = P_A_BYTES + P_B_BYTES;
constexpr int U_A_BYTES = BM * BKE;        // 16 KiB
constexpr int U_B_BYTES = BN * BKE;        // 32 KiB
constexpr int U_STAGE = U_A_BYTES + U_B_BYTES;
constexpr int UNPACK_WARPS = 12;           // one thread per packed row of a stage (128 + 256)
constexpr int EPI_WARPS = 4;
constexpr int WARP_PRODUCER = 0, WARP_MMA = 1, WARP_UNPACK0 = 2, WARP_EPI0 = WARP_UNPACK0 + UNPACK_WARPS;
constexpr int THREADS = (WARP_EPI0 + EPI_WARPS) * 32;   // 576
constexpr int TMEM_COLS = 2 * BN;          // two accumulators
constexpr int NUM_BARS = 2 * PSTAGES + 2 * USTAGES + 2 * 2 + 1;
// Per-tile epilogue column parameters, one private copy per epilogue warp:
// float4 {alpha, gamma, beta, -} and int2 {c1, len2} of the threshold test
// per column.
constexpr int COLP_BYTES = EPI_WARPS * BN * (16 + 8);
constexpr int SMEM_FIXED = USTAGES * U_STAGE + COLP_BYTES + NUM_BARS * 8 + 16 + 1024;
constexpr int SMEM_BYTES = SMEM_FIXED + PSTAGES * P_STAGE;
// Shared memory one CTA may use on sm_100 (opt-in maximum).
constexpr int SMEM_LIMIT = 227 * 1024;
// Bit planes per operand row in the plane-code mode (unsigned codes of up to
// this many bits), and bases per operand in the bases mode.
constexpr int MAX_CODE_PLANES = 4;
constexpr int MAX_BASES = 8;
// kind::i8 instruction descriptor: D s32 (bits 4-5 = 2), A and B type at bits
// 7-9 and 10-12 (1 = s8, 0 = u8), both K-major, N >> 3 at bits 17-22, M >> 4
// at 24-28.
constexpr uint32_t IDESC = (2u << 4) | (1u << 7) | (1u << 10) | ((uint32_t)(BN >> 3) << 17) |
                           ((uint32_t)(BM >> 4) << 24);
constexpr uint32_t IDESC_U8 = (2u << 4) | ((uint32_t)(BN >> 3) << 17) | ((uint32_t)(BM >> 4) << 24);

// Bytes of one packed stage and the packed-ring depth that fits beside the
// fixed part of shared memory.  Binary and bases modes: 128 + 256 packed rows
// of 16 bytes.  Plane-code mode: every code row brings its planes.
__host__ __device__ constexpr int packed_stage_bytes(int mode, int ja, int jw) {
    return mode == 1 ? (BM * ja + BN * jw) * 16 : P_STAGE;
}
__host__ __device__ constexpr int packed_stages(int mode, int ja, int jw) {
    return (SMEM_LIMIT - SMEM_FIXED) / packed_stage_bytes(mode, ja, jw) < PSTAGES
               ? (SMEM_LIMIT - SMEM_FIXED) / packed_stage_bytes(mode, ja, jw)
               : PSTAGES;
}
}  // namespace tc

// Kernel modes of xnor_gemm_tc_kernel.
//  TC_BINARY      +1/-1 operands, one packed row per matrix row (eq. (6)).
//  TC_PLANE_CODES unsigned integer codes stored as bit planes: plane p of
//                 code row r is packed row r * planes + p; the unpack folds
//                 the planes into one byte per element, code = sum_p bit_p
//                 2^p, and the tensor cores multiply u8 x u8 -- the whole
//                 multi-bit product sum_k a_k w_k in one pass (DoReFa-Net's
//                 bit-convolution).
//  TC_BASES       +1/-1 binary bases stored plane-interleaved the same way;
//                 each base is expanded like a binary row, so every pair
//                 (base j of A, base i of W) gets its own +1/-1 product, and
//                 the epilogue forms sum_j beta_j sum_i alpha_i[n] * s_ji
//                 (ABC-Net).
enum TcMode { TC_BINARY = 0, TC_PLANE_CODES = 1, TC_BASES = 2 };

// Plane layout and the bases epilogue's parameters.
struct TcPlanes {
    int ja, jw;           // planes per A / W row inside a stage (bases: padded to a power of two)
    int j_real, i_real;   // bases actually present (the padded ones are zero-filled by the TMA box)
    int pstages;          // packed-ring depth
    int p_stage;          // bytes per packed stage
    const float* beta;    // bases: beta_j, [j_real]
    const float* alpha;   // bases: alpha_i[n], [i_real][lda_alpha]
    int64_t lda_alpha;
    float* y;             // bases: fp32 output [M, N]
    int64_t ldy;
};

// Shared-memory matrix descriptor for a K-major, 128B-swizzled operand tile
// whose rows are 128 bytes (8-row groups 1024 bytes apart): start address,
// leading offset 16 B (unused for this layout), stride offset 1024 B,
// descriptor version 1, layout type 2 (SWIZZLE_128B).
__device__ __forceinline__ uint64_t umma_desc_sw128(uint32_t smem_addr) {
    return (uint64_t)((smem_addr >> 4) & 0x3FFFu) | ((uint64_t)1u << 16) | ((uint64_t)(1024u >> 4) << 32) |
           ((uint64_t)1u << 46) | ((uint64_t)2u << 61);
}

__device__ __forceinline__ void tc_fence_before() { asm volatile("tcgen05.fence::before_thread_sync;" ::: "memory"); }
__device__ __forceinline__ void tc_fence_after() { asm volatile("tcgen05.fence::after_thread_sync;" ::: "memory"); }

__device__ __forceinline__ void tmem_alloc(uint32_t* dst, uint32_t ncols) {
    asm volatile("tcgen05.alloc.cta_group::1.sync.aligned.shared::cta.b32 [%0], %1;" ::"r"(smem_u32(dst)),
                 "r"(ncols)
                 : "memory");
}
__device__ __forceinline__ void tmem_relinquish() {
    asm volatile("tcgen05.relinquish_alloc_permit.cta_group::1.sync.aligned;" ::: "memory");
}
__device__ __forceinline__ void tmem_dealloc(uint32_t taddr, uint32_t ncols) {
    asm volatile("tcgen05.dealloc.cta_group::1.sync.aligned.b32 %0, %1;" ::"r"(taddr), "r"(ncols) : "memory");
}

__device__ __forceinline__ void mma_i8(uint32_t d_tmem, uint64_t adesc, uint64_t bdesc, uint32_t idesc,
                                       uint32_t accumulate) {
    asm volatile(
        "{\n\t.reg .pred p;\n\t"
        "setp.ne.b32 p, %4, 0;\n\t"
        "tcgen05.mma.cta_group::1.kind::i8 [%0], %1, %2, %3, p;\n\t}" ::"r"(d_tmem),
        "l"(adesc), "l"(bdesc), "r"(idesc), "r"(accumulate)
        : "memory");
}

// Arrive on `bar` once every tcgen05.mma issued so far by this thread is done.
__device__ __forceinline__ void mma_commit(uint64_t* bar) {
    asm volatile("tcgen05.commit.cta_group::1.mbarrier::arrive::one.shared::cluster.b64 [%0];" ::"r"(smem_u32(bar))
                 : "memory");
}

// TMEM -> registers for one warp: 32 lanes x 32 (or 16) consecutive 32-bit
// columns, followed by tcgen05.wait::ld in the SAME asm statement.  The load
// is asynchronous: its destination registers hold the values only after the
// wait.  With the wait in a separate asm statement nothing ties the uses of
// those registers to it (the wait names no register), so the compiler may
// schedule arithmetic on them before the wait and read stale values.
// Keeping both instructions in one statement defines the outputs at the end
// of the statement, after the wait.
__device__ __forceinline__ void tmem_ld32_sync(uint32_t taddr, uint32_t (&r)[32]) {
    asm volatile(
        "tcgen05.ld.sync.aligned.32x32b.x32.b32 "
        "{%0, %1, %2, %3, %4, %5, %6, %7, %8, %9, %10, %11, %12, %13, %14, %15, "
        "%16, %17, %18, %19, %20, %21, %22, %23, %24, %25, %26, %27, %28, %29, %30, %31}, [%32];\n\t"
        "tcgen05.wait::ld.sync.aligned;"
        : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3]), "=r"(r[4]), "=r"(r[5]), "=r"(r[6]), "=r"(r[7]),
          "=r"(r[8]), "=r"(r[9]), "=r"(r[10]), "=r"(r[11]), "=r"(r[12]), "=r"(r[13]), "=r"(r[14]), "=r"(r[15]),
          "=r"(r[16]), "=r"(r[17]), "=r"(r[18]), "=r"(r[19]), "=r"(r[20]), "=r"(r[21]), "=r"(r[22]), "=r"(r[23]),
          "=r"(r[24]), "=r"(r[25]), "=r"(r[26]), "=r"(r[27]), "=r"(r[28]), "=r"(r[29]), "=r"(r[30]), "=r"(r[31])
        : "r"(taddr)
        : "memory");
}
__device__ __forceinline__ void tmem_ld16_sync(uint32_t taddr, uint32_t (&r)[16]) {
    asm volatile(
        "tcgen05.ld.sync.aligned.32x32b.x16.b32 "
        "{%0, %1, %2, %3, %4, %5, %6, %7, %8, %9, %10, %11, %12, %13, %14, %15}, [%16];\n\t"
        "tcgen05.wait::ld.sync.aligned;"
        : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3]), "=r"(r[4]), "=r"(r[5]), "=r"(r[6]), "=r"(r[7]),
          "=r"(r[8]), "=r"(r[9]), "=r"(r[10]), "=r"(r[11]), "=r"(r[12]), "=r"(r[13]), "=r"(r[14]), "=r"(r[15])
        : "r"(taddr)
        : "memory");
}

constexpr int log2_pow2(int v) { return v <= 1 ? 0 : 1 + log2_pow2(v >> 1); }

// Binary bases, one 32-column accumulator chunk of one thread (lane jl of
// the JA lanes of its output row; JW accumulator columns per output column,
// so the chunk covers G = 32 / JW output columns).  acc holds s + pad for
// each base pair (s the +1/-1 product, pad the +1 K padding) as int32
// (INT_ACC, the int8 kernel) or as an fp32 integer (the e2m1 kernel); s
// is exact either way.  v_o = sum_i alpha_i[n_o] s_ji (fused multiply-adds
// in i order), times beta_j; the JA lanes of the row then add their v by a
// reduce-scatter, low lane bit first: at each step a lane keeps one half of
// its values, hands the other half to its partner and adds the partner's
// half of its own, so the adds pair up exactly as a butterfly would, but a
// row's outputs end up spread over its lanes (P = G / JA consecutive ones
// each) after G (1 - 1 / JA) shuffles instead of G log2 JA.  With G < JA the
// last steps are a butterfly and the lowest lane of each group stores.
// Shared-memory reads (the chunk's 32 alphas as eight broadcast 16-byte
// loads) and shuffles share the shared-memory pipe with the unpack warps'
// stores and the MMAs' operand reads, so the epilogue keeps both few.
template <int JA, int JW, bool INT_ACC>
__device__ __forceinline__ void bases_combine_chunk(const uint32_t (&acc)[32], const float* ca, int pad, float bj,
                                                    int jl, float* yrow, int nb, int N, bool vec) {
    constexpr int G = 32 / JW;
    constexpr int LOG_JA = log2_pow2(JA), LOG_G = log2_pow2(G);
    constexpr int SCAT = LOG_JA < LOG_G ? LOG_JA : LOG_G;
    constexpr int P = G >> SCAT;
    float v[G];
    #pragma unroll
    for (int g = 0; g < G; ++g) v[g] = 0.0f;
    #pragma unroll
    for (int q = 0; q < 8; ++q) {
        const float4 a = reinterpret_cast<const float4*>(ca)[q];
        const float av[4] = {a.x, a.y, a.z, a.w};
        #pragma unroll
        for (int e = 0; e < 4; ++e) {
            const int col = 4 * q + e;
            const float s = INT_ACC ? (float)((int32_t)acc[col] - pad) : __uint_as_float(acc[col]) - (float)pad;
            v[col / JW] = fmaf(av[e], s, v[col / JW]);
        }
    }
    #pragma unroll
    for (int g = 0; g < G; ++g) v[g] *= bj;
    int o0 = 0;                                       // first output column (of the chunk) this lane keeps
    #pragma unroll
    for (int s = 0; s < SCAT; ++s) {
        const int half = G >> (s + 1);
        const bool up = ((jl >> s) & 1) != 0;
        #pragma unroll
        for (int h = 0; h < half; ++h) {
            const float send = up ? v[h] : v[h + half];
            const float keep = up ? v[h + half] : v[h];
            v[h] = keep + __shfl_xor_sync(0xffffffffu, send, 1 << s);
        }
        if (up) o0 += half;
    }
    #pragma unroll
    for (int s = SCAT; s < LOG_JA; ++s) v[0] += __shfl_xor_sync(0xffffffffu, v[0], 1 << s);
    if ((jl >> SCAT) != 0 || yrow == nullptr) return;
    const int n = nb + o0;
    constexpr int VW = P < 4 ? P : 4;
    if (vec && VW > 1 && n + P <= N && (n & (VW - 1)) == 0) {
        #pragma unroll
        for (int p = 0; p < P; p += VW) {
            if constexpr (VW == 4) *reinterpret_cast<float4*>(yrow + n + p) = make_float4(v[p], v[p + 1], v[p + 2], v[p + 3]);
            else if constexpr (VW == 2) *reinterpret_cast<float2*>(yrow + n + p) = make_float2(v[p], v[p + 1]);
        }
    } else {
        #pragma unroll
        for (int p = 0; p < P; ++p)
            if (n + p < N) yrow[n + p] = v[p];
    }
}

// Dispatch of bases_combine_chunk over (log2 ja, log2 jw), both 0..3; the
// shape is the same for the whole launch.
template <bool INT_ACC>
__device__ __forceinline__ void bases_combine(int shape, const uint32_t (&acc)[32], const float* ca, int pad, float bj,
                                              int jl, float* yrow, int nb, int N, bool vec) {
    switch (shape) {
#define BNN_BASES_CASE(LA, LW)                                                                        \
    case (LA) * 4 + (LW):                                                                             \
        bases_combine_chunk<1 << (LA), 1 << (LW), INT_ACC>(acc, ca, pad, bj, jl, yrow, nb, N, vec);   \
        break;
        BNN_BASES_CASE(0, 0) BNN_BASES_CASE(0, 1) BNN_BASES_CASE(0, 2) BNN_BASES_CASE(0, 3)
        BNN_BASES_CASE(1, 0) BNN_BASES_CASE(1, 1) BNN_BASES_CASE(1, 2) BNN_BASES_CASE(1, 3)
        BNN_BASES_CASE(2, 0) BNN_BASES_CASE(2, 1) BNN_BASES_CASE(2, 2) BNN_BASES_CASE(2, 3)
        BNN_BASES_CASE(3, 0) BNN_BASES_CASE(3, 1) BNN_BASES_CASE(3, 2) BNN_BASES_CASE(3, 3)
#undef BNN_BASES_CASE
        default: break;
    }
}

// Bounded wait that also gives up as soon as another role of the CTA aborted.
__device__ __forceinline__ bool tc_wait(uint64_t* bar, uint32_t parity, volatile int* abort_flag) {
    if (mbar_try_wait(bar, parity)) return true;
    const unsigned long long t0 = globaltimer_ns();
    while (true) {
        #pragma unroll 1
        for (int i = 0; i < 32; ++i)
            if (mbar_try_wait(bar, parity)) return true;
        if (*abort_flag) return false;
        if (globaltimer_ns() - t0 > kWaitTimeoutNs) {
            flag_device_error(BNN_ERR_DEVICE_TIMEOUT);
            *abort_flag = 1;
            return false;
        }
    }
}

// 32 sign bits -> 32 signed bytes (+1 / -1), as two 16-byte chunks.
// Register s (0..7) of the 32 bytes holds elements 7-s, 15-s, 23-s and 31-s:
// shifting the word left by s puts those bits at the sign positions of its 4
// bytes, a PRMT with sign-replicating selectors turns each byte into 0x00 or
// 0xFF, and one LOP3 maps 0x00 -> 0x01 (+1), 0xFF -> 0xFF (-1).  Three
// operations per 4 bytes.  The element order inside a word's 32 bytes is
// therefore a fixed permutation; both operands of a product are expanded by
// this same function, so every K-sum pairs the same elements.
__device__ __forceinline__ void expand_word_pm1(uint32_t w, uint4& c0, uint4& c1) {
    uint32_t r[8];
    #pragma unroll
    for (int s = 0; s < 8; ++s) {
        uint32_t m;
        asm("prmt.b32 %0, %1, 0, 0xBA98;" : "=r"(m) : "r"(w << s));
        r[s] = (m & 0xFEFEFEFEu) | 0x01010101u;
    }
    c0 = make_uint4(r[0], r[1], r[2], r[3]);
    c1 = make_uint4(r[4], r[5], r[6], r[7]);
}

// Bit planes -> unsigned byte codes.  `w[p]` holds word q of plane p (the
// same 32 elements in every plane); byte e of the result is sum_p bit_p(e)
// 2^p.  Per plane and 4 bytes: a shift, a sign-replicating PRMT (byte ->
// 0x00 / 0xFF as in expand_word_pm1) and one LOP3 that keeps bit p of each
// byte and ORs it in.  The byte order inside the 32 is expand_word_pm1's
// permutation, so an A row and a W row expanded by this function pair the
// same elements.
__device__ __forceinline__ void expand_planes_u8(const uint32_t (&w)[tc::MAX_CODE_PLANES], int planes, uint4& c0,
                                                 uint4& c1) {
    uint32_t r[8];
    #pragma unroll
    for (int s = 0; s < 8; ++s) r[s] = 0u;
    #pragma unroll
    for (int p = 0; p < tc::MAX_CODE_PLANES; ++p) {
        if (p < planes) {
            const uint32_t wp = w[p], mask = 0x01010101u << p;
            #pragma unroll
            for (int s = 0; s < 8; ++s) {
                uint32_t m;
                asm("prmt.b32 %0, %1, 0, 0xBA98;" : "=r"(m) : "r"(wp << s));
                asm("lop3.b32 %0, %1, %2, %3, 0xf8;" : "=r"(r[s]) : "r"(r[s]), "r"(m), "r"(mask));   // r | (m & mask)
            }
        }
    }
    c0 = make_uint4(r[0], r[1], r[2], r[3]);
    c1 = make_uint4(r[4], r[5], r[6], r[7]);
}

// Hand a packed stage back to the TMA producer once this warp has read it.
// The reads are generic-proxy loads; the producer's next fill of the same
// bytes is an async-proxy (TMA) write issued as soon as the stage's "empty"
// barrier completes.  The proxy fence orders this thread's reads before any
// later async-proxy access, so the fill cannot land before a read it would
// overwrite has taken its value (without it, full-output comparisons caught
// unpack warps expanding words of a later stage).
__device__ __forceinline__ void release_packed_stage(uint64_t* empty_bar, int lane) {
    fence_proxy_async_shared();
    __syncwarp();
    if (lane == 0) mbar_arrive(empty_bar);
}

template <int MODE>
__global__ void __launch_bounds__(tc::THREADS, 1)
xnor_gemm_tc_kernel(const __grid_constant__ CUtensorMap tmA, const __grid_constant__ CUtensorMap tmW, int M, int N,
                    int K, int kw, int tiles_m, int tiles_n, GemmEpilogue ep, TcPlanes pl) {
    using namespace tc;
    extern __shared__ uint8_t smem_raw[];
    // Packed-ring geometry: fixed in the binary and bases modes, set by the
    // plane counts in the plane-code mode.
    const int pst = MODE == TC_PLANE_CODES ? pl.pstages : PSTAGES;
    const int pstage = MODE == TC_PLANE_CODES ? pl.p_stage : P_STAGE;
    const int pa_bytes = MODE == TC_PLANE_CODES ? BM * pl.ja * 16 : P_A_BYTES;
    // Rows (and columns) of the output per tile: the bases mode spends ja (jw)
    // accumulator lanes (columns) on each output row (column).
    const int rows_per_tile = MODE == TC_BASES ? BM / pl.ja : BM;
    const int cols_per_tile = MODE == TC_BASES ? BN / pl.jw : BN;
    // 1024-byte aligned base, derived by offset from the __shared__ array so
    // that the compiler keeps every access in the shared address space.
    uint8_t* smem = smem_raw + ((1024u - (smem_u32(smem_raw) & 1023u)) & 1023u);
    uint8_t* uring = smem;                                   // USTAGES x (A 16 KiB | W 32 KiB)
    uint8_t* pring = smem + USTAGES * U_STAGE;               // pst x (A | W packed)
    float4* colf = reinterpret_cast<float4*>(pring + pst * pstage);           // [EPI_WARPS][BN]
    int2* colt = reinterpret_cast<int2*>(colf + EPI_WARPS * BN);               // [EPI_WARPS][BN]
    uint64_t* bars = reinterpret_cast<uint64_t*>(colt + EPI_WARPS * BN);
    uint64_t* pfull = bars;
    uint64_t* pempty = pfull + PSTAGES;
    uint64_t* ufull = pempty + PSTAGES;
    uint64_t* uempty = ufull + USTAGES;
    uint64_t* afull = uempty + USTAGES;
    uint64_t* aempty = afull + 2;
    uint64_t* drain = aempty + 2;
    uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(drain + 1);
    volatile int* abort_flag = reinterpret_cast<volatile int*>(tmem_slot + 1);

    const int warp = threadIdx.x >> 5;
    const int lane = threadIdx.x & 31;
    const int nk = kw / BKW;                                  // kw is a multiple of 4
    const int tiles = tiles_m * tiles_n;

    if (threadIdx.x == 0) {
        prefetch_tensormap(&tmA);
        prefetch_tensormap(&tmW);
        for (int s = 0; s < pst; ++s) {
            mbar_init(&pfull[s], 1);
            mbar_init(&pempty[s], UNPACK_WARPS);
        }
        for (int s = 0; s < USTAGES; ++s) {
            mbar_init(&ufull[s], UNPACK_WARPS);
            mbar_init(&uempty[s], 1);
        }
        for (int b = 0; b < 2; ++b) {
            mbar_init(&afull[b], 1);
            mbar_init(&aempty[b], EPI_WARPS);
        }
        mbar_init(drain, 1);
        *abort_flag = 0;
        fence_mbarrier_init();
    }
    if (warp == WARP_MMA) {
        tmem_alloc(tmem_slot, TMEM_COLS);
        tmem_relinquish();
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem_base = *tmem_slot;

    if (warp == WARP_PRODUCER) {
        // ------------------------------ TMA producer ------------------------------
        if (lane == 0) {
            uint32_t g = 0, issued = 0;
            bool ok = true;
            for (int t = blockIdx.x; ok && t < tiles; t += gridDim.x) {
                const int m0 = (t / tiles_n) * rows_per_tile, n0 = (t % tiles_n) * cols_per_tile;
                for (int ks = 0; ks < nk; ++ks, ++g) {
                    const uint32_t s = g % (uint32_t)pst;
                    if (g >= (uint32_t)pst && !tc_wait(&pempty[s], ((g / pst) - 1) & 1, abort_flag)) { ok = false; break; }
                    uint8_t* dst = pring + s * pstage;
                    mbar_arrive_expect_tx(&pfull[s], pstage);
                    if constexpr (MODE == TC_BINARY) {
                        tma_load_2d(dst, &tmA, ks * BKW, m0, &pfull[s]);
                        tma_load_2d(dst + pa_bytes, &tmW, ks * BKW, n0, &pfull[s]);
                    } else {
                        // Boxes of {4 words, all planes, rows}: the planes of
                        // a row land next to each other, 16 bytes apart.
                        tma_load_3d(dst, &tmA, ks * BKW, 0, m0, &pfull[s]);
                        tma_load_3d(dst + pa_bytes, &tmW, ks * BKW, 0, n0, &pfull[s]);
                    }
                    ++issued;
                }
            }
            // Let the copies still in flight land before the CTA can retire
            // (also after an abort).
            for (uint32_t q = issued > (uint32_t)pst ? issued - pst : 0; q < issued; ++q)
                if (!mbar_wait_bounded(&pfull[q % pst], (q / pst) & 1)) break;
        }
    } else if (warp == WARP_MMA) {
        // ------------------------------ MMA issuer ------------------------------
        if (lane == 0) {
            uint32_t g = 0;
            int lt = 0;
            bool ok = true;
            const uint32_t ubase = smem_u32(uring);
            const uint32_t idesc = MODE == TC_PLANE_CODES ? IDESC_U8 : IDESC;
            for (int t = blockIdx.x; ok && t < tiles; t += gridDim.x, ++lt) {
                const int b = lt & 1;
                if (lt >= 2 && !tc_wait(&aempty[b], ((lt >> 1) - 1) & 1, abort_flag)) break;
                tc_fence_after();
                const uint32_t d_tmem = tmem_base + (uint32_t)(b * BN);
                for (int ks = 0; ks < nk; ++ks, ++g) {
                    const uint32_t s = g % USTAGES;
                    if (!tc_wait(&ufull[s], (g / USTAGES) & 1, abort_flag)) { ok = false; break; }
                    tc_fence_after();
                    const uint32_t a_addr = ubase + s * U_STAGE;
                    const uint32_t b_addr = a_addr + U_A_BYTES;
                    #pragma unroll
                    for (int kk = 0; kk < BKE / UMMA_K; ++kk) {
                        // Advancing the start address by 32 B steps through K inside the swizzle atom.
                        mma_i8(d_tmem, umma_desc_sw128(a_addr + kk * UMMA_K), umma_desc_sw128(b_addr + kk * UMMA_K),
                               idesc, (ks | kk) != 0 ? 1u : 0u);
                    }
                    mma_commit(&uempty[s]);
                }
                if (ok) mma_commit(&afull[b]);
            }
            // Every MMA issued above is complete once this arrives (waited for
            // even after an abort: TMEM is freed only after the last MMA).
            mma_commit(drain);
            mbar_wait_bounded(drain, 0);
        }
        __syncwarp();
    } else if (warp < WARP_EPI0) {
        // ------------------------------ unpack warps ------------------------------
        // Thread u expands row u of the stage (A rows 0..127, then W rows) into
        // 128 bytes: one 16-byte load of its 4 words per plane, eight 16-byte
        // stores.  Binary and bases modes: a row is one +1/-1 plane.  Plane-code
        // mode: a row is a code row whose planes sit 16 bytes apart.
        const int u = threadIdx.x - WARP_UNPACK0 * 32;               // 0..383
        const bool is_a = u < BM;
        const int r = is_a ? u : u - BM;
        const int sw = r & 7;
        const int planes = MODE == TC_PLANE_CODES ? (is_a ? pl.ja : pl.jw) : 1;
        uint32_t g = 0;
        bool ok = true;
        for (int t = blockIdx.x; ok && t < tiles; t += gridDim.x) {
            for (int ks = 0; ks < nk; ++ks, ++g) {
                const uint32_t ps = g % (uint32_t)pst, us = g % USTAGES;
                bool w1 = tc_wait(&pfull[ps], (g / pst) & 1, abort_flag);
                bool w2 = w1 && (g < USTAGES || tc_wait(&uempty[us], ((g / USTAGES) - 1) & 1, abort_flag));
                if (!__all_sync(0xffffffffu, w1 && w2)) { ok = false; break; }
                uint8_t* row = uring + us * U_STAGE + (is_a ? 0 : U_A_BYTES) + r * 128;
                if constexpr (MODE == TC_PLANE_CODES) {
                    const uint8_t* src = pring + ps * pstage + (is_a ? 0 : pa_bytes) + r * planes * 16;
                    uint32_t wq[4][MAX_CODE_PLANES];
                    #pragma unroll
                    for (int p = 0; p < MAX_CODE_PLANES; ++p) {
                        const uint4 pk = p < planes ? *reinterpret_cast<const uint4*>(src + p * 16)
                                                    : make_uint4(0u, 0u, 0u, 0u);
                        wq[0][p] = pk.x; wq[1][p] = pk.y; wq[2][p] = pk.z; wq[3][p] = pk.w;
                    }
                    release_packed_stage(&pempty[ps], lane);
                    #pragma unroll
                    for (int q = 0; q < 4; ++q) {
                        uint4 c0, c1;
                        expand_planes_u8(wq[q], planes, c0, c1);
                        *reinterpret_cast<uint4*>(row + (((2 * q) ^ sw) << 4)) = c0;
                        *reinterpret_cast<uint4*>(row + (((2 * q + 1) ^ sw) << 4)) = c1;
                    }
                } else {
                    const uint4 pk = *reinterpret_cast<const uint4*>(pring + ps * pstage + u * 16);
                    release_packed_stage(&pempty[ps], lane);
                    const uint32_t wq[4] = {pk.x, pk.y, pk.z, pk.w};
                    #pragma unroll
                    for (int q = 0; q < 4; ++q) {
                        uint4 c0, c1;
                        expand_word_pm1(wq[q], c0, c1);
                        *reinterpret_cast<uint4*>(row + (((2 * q) ^ sw) << 4)) = c0;
                        *reinterpret_cast<uint4*>(row + (((2 * q + 1) ^ sw) << 4)) = c1;
                    }
                }
                fence_proxy_async_shared();                           // make the bytes visible to the tensor core
                __syncwarp();
                if (lane == 0) mbar_arrive(&ufull[us]);
            }
        }
    } else if constexpr (MODE != TC_BASES) {
        // ------------------------------ epilogue warps ------------------------------
        // Per tile, each epilogue warp first stages the tile's column parameters
        // in its own shared-memory copy (alpha/gamma/beta and the threshold test
        // as one unsigned range check on the raw accumulator), then each thread
        // turns its row's 256 accumulators into outputs with broadcast shared
        // loads instead of per-column global loads.  The copy is private to
        // the warp, so only __syncwarp orders it and no warp waits for
        // another.
        const int quad = warp & 3;                                    // TMEM lanes 32*quad .. 32*quad + 31
        float4* wcolf = colf + (warp - WARP_EPI0) * BN;
        int2* wcolt = colt + (warp - WARP_EPI0) * BN;
        const int kp = nk * BKE;                                      // padded K: acc = kp - 2 * popcount
        // Binary: (+1)(+1) pad positions per output.  Plane codes: a pad
        // element is code 0 and adds nothing.
        const int pad = MODE == TC_PLANE_CODES ? 0 : kp - K;
        const bool affine = ep.gamma != nullptr;
        int lt = 0;
        for (int t = blockIdx.x; t < tiles; t += gridDim.x, ++lt) {
            const int b = lt & 1;
            const int m0 = (t / tiles_n) * BM, n0 = (t % tiles_n) * BN;
            // Stage this tile's columns once every lane of the warp is done
            // with the previous tile's copy.
            __syncwarp();
            for (int i = lane; i < BN; i += 32) {
                const int n = n0 + i;
                float4 f = make_float4(0.f, 1.f, 0.f, 0.f);
                int2 th = make_int2(0, 0);                            // len2 = 0: bit never set
                if (n < N) {
                    if (ep.alpha != nullptr) f.x = __ldg(ep.alpha + n);
                    if (affine) { f.y = __ldg(ep.gamma + n); f.z = __ldg(ep.beta + n); }
                    if (ep.c_bits != nullptr) {
                        // d = popcount = (kp - acc) / 2 lies in [0, K].  mode 0: bit = d > T,
                        // the interval [max(T+1, 0), K]; mode 1: bit = d < T, the interval
                        // [0, min(T-1, K)]; other modes: empty.  With lo and len of the
                        // interval, bit = (unsigned)(d - lo) < len, which is
                        // (unsigned)(c1 - acc) < 2*len for c1 = kp - 2*lo (kp - acc is even).
                        const long long T = __ldg(ep.thresh + n);
                        const int md = ep.thresh_mode[n];
                        long long lo = 0, len = 0;
                        if (md == 0) {
                            lo = T + 1 > 0 ? T + 1 : 0;
                            len = K - lo + 1 > 0 ? K - lo + 1 : 0;
                        } else if (md == 1) {
                            len = T < K + 1 ? T : K + 1;
                            if (len < 0) len = 0;
                        }
                        th = make_int2((int)(uint32_t)(kp - 2 * lo), (int)(uint32_t)(2 * len));
                    }
                }
                wcolf[i] = f;
                wcolt[i] = th;
            }
            __syncwarp();
            if (!__all_sync(0xffffffffu, tc_wait(&afull[b], (lt >> 1) & 1, abort_flag))) break;
            tc_fence_after();
            const int m = m0 + 32 * quad + lane;
            const float4* cf = wcolf;
            const int2* ct = wcolt;
            #pragma unroll 1
            for (int c = 0; c < BN / 32; ++c) {
                uint32_t r[32];
                tmem_ld32_sync(tmem_base + ((uint32_t)(32 * quad) << 16) + (uint32_t)(b * BN + 32 * c), r);
                if (c == BN / 32 - 1) {
                    // Whole accumulator read: hand it back to the MMA warp.
                    tc_fence_before();
                    __syncwarp();
                    if (lane == 0) mbar_arrive(&aempty[b]);
                }
                const int nb = n0 + 32 * c;
                if (nb >= N) {
                    // Past the last column: a packed output still has pad words here.
                    if (ep.c_bits != nullptr && m < M && nb / 32 < ep.bits_words)
                        ep.c_bits[(int64_t)m * ep.ldb + nb / 32] = 0u;
                    continue;
                }
                const bool full_chunk = nb + 32 <= N;
                if (ep.c_bits != nullptr) {
                    uint32_t word = 0;
                    #pragma unroll
                    for (int j = 0; j < 32; ++j) {
                        const int2 q = ct[32 * c + j];
                        word |= ((uint32_t)(q.x - (int32_t)r[j]) < (uint32_t)q.y ? 1u : 0u) << j;
                    }
                    if (m < M && nb / 32 < ep.bits_words) ep.c_bits[(int64_t)m * ep.ldb + nb / 32] = word;
                }
                if (m < M && ep.c_i32 != nullptr) {
                    int32_t* dst = ep.c_i32 + (int64_t)m * ep.ldc + nb;
                    const bool vec = full_chunk && ((reinterpret_cast<uintptr_t>(dst) & 15) == 0);
                    #pragma unroll
                    for (int j = 0; j < 32; j += 4) {
                        const int4 o = make_int4((int32_t)r[j] - pad, (int32_t)r[j + 1] - pad,
                                                 (int32_t)r[j + 2] - pad, (int32_t)r[j + 3] - pad);
                        if (vec) {
                            *reinterpret_cast<int4*>(dst + j) = o;
                        } else {
                            if (nb + j < N) dst[j] = o.x;
                            if (nb + j + 1 < N) dst[j + 1] = o.y;
                            if (nb + j + 2 < N) dst[j + 2] = o.z;
                            if (nb + j + 3 < N) dst[j + 3] = o.w;
                        }
                    }
                }
                if (m < M && ep.c_f32 != nullptr) {
                    float* dst = ep.c_f32 + (int64_t)m * ep.ldf + nb;
                    const bool vec = full_chunk && ((reinterpret_cast<uintptr_t>(dst) & 15) == 0);
                    #pragma unroll
                    for (int j = 0; j < 32; j += 4) {
                        float y[4];
                        #pragma unroll
                        for (int k = 0; k < 4; ++k) {
                            const float4 f = cf[32 * c + j + k];
                            float v = f.x * (float)((int32_t)r[j + k] - pad);
                            if (affine) v = fmaf(f.y, v, f.z);
                            y[k] = v;
                        }
                        if (vec) {
                            *reinterpret_cast<float4*>(dst + j) = make_float4(y[0], y[1], y[2], y[3]);
                        } else {
                            #pragma unroll
                            for (int k = 0; k < 4; ++k)
                                if (nb + j + k < N) dst[j + k] = y[k];
                        }
                    }
                }
            }
            // The last column tile also zeroes pad words of the packed output that no tile covers.
            if (ep.c_bits != nullptr && (t % tiles_n) == tiles_n - 1 && m < M) {
                for (int64_t wd = (int64_t)(n0 + BN) / 32; wd < ep.bits_words; ++wd)
                    ep.c_bits[(int64_t)m * ep.ldb + wd] = 0u;
            }
        }
    } else {
        // ------------------------- epilogue warps, bases mode -------------------------
        // Accumulator lane L holds base j = L mod ja of output row L / ja;
        // column c holds base i = c mod jw of output column c / jw.
        // bases_combine forms each output from its ja x jw accumulators.
        // Padded bases have beta_j = 0 or alpha_i[n] = 0, so their products
        // add exactly 0.
        const int quad = warp & 3;
        const int ja = pl.ja, jw = pl.jw;
        float* wcola = reinterpret_cast<float*>(colf + (warp - WARP_EPI0) * BN);   // alpha per column
        const int kp = nk * BKE;
        const int pad = kp - K;
        const int L = 32 * quad + lane;
        const int jl = L & (ja - 1);
        const float bj = jl < pl.j_real ? __ldg(pl.beta + jl) : 0.0f;
        const int outs_per_chunk = 32 / jw;                           // output columns per 32 accumulator columns
        const int shape = log2_pow2(ja) * 4 + log2_pow2(jw);
        const bool vec = ((reinterpret_cast<uintptr_t>(pl.y) | ((uintptr_t)pl.ldy * 4u)) & 15u) == 0;
        int lt = 0;
        for (int t = blockIdx.x; t < tiles; t += gridDim.x, ++lt) {
            const int b = lt & 1;
            const int m0 = (t / tiles_n) * rows_per_tile, n0 = (t % tiles_n) * cols_per_tile;
            __syncwarp();
            for (int i = lane; i < BN; i += 32) {
                const int n = n0 + i / jw, ib = i & (jw - 1);
                wcola[i] = (n < N && ib < pl.i_real) ? __ldg(pl.alpha + (int64_t)ib * pl.lda_alpha + n) : 0.0f;
            }
            __syncwarp();
            if (!__all_sync(0xffffffffu, tc_wait(&afull[b], (lt >> 1) & 1, abort_flag))) break;
            tc_fence_after();
            const int m = m0 + L / ja;
            #pragma unroll 1
            for (int c = 0; c < BN / 32; ++c) {
                uint32_t r[32];
                tmem_ld32_sync(tmem_base + ((uint32_t)(32 * quad) << 16) + (uint32_t)(b * BN + 32 * c), r);
                if (c == BN / 32 - 1) {
                    tc_fence_before();
                    __syncwarp();
                    if (lane == 0) mbar_arrive(&aempty[b]);
                }
                const int nb = n0 + c * outs_per_chunk;
                if (nb >= N) continue;                                // uniform across the warp
                float* yrow = m < M ? pl.y + (int64_t)m * pl.ldy : nullptr;
                bases_combine<true>(shape, r, wcola + 32 * c, pad, bj, jl, yrow, nb, N, vec);
            }
        }
    }

    // ------------------------------ teardown ------------------------------
    tc_fence_before();
    __syncthreads();
    if (warp == WARP_MMA) {
        tc_fence_after();
        tmem_dealloc(tmem_base, TMEM_COLS);
    }
}

}  // namespace bnn
