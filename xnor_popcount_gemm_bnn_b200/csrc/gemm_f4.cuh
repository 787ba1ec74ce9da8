// Packed binary GEMM on the tensor cores with 4-bit operands
// (tcgen05.mma kind::mxf4, e2m1 elements, unit block scales).
//
// Same product as gemm_popc.cuh and gemm_tc.cuh -- s[m, n] = sum_k a_mk w_nk
// over +1/-1 values ("Extreme Quantization: Binary, Ternary & 1-bit LLMs",
// eq. (1), (4) and (6)).  +1 and -1 are exact e2m1 values (0x2 and 0xA: the
// sign bit is bit 3 of the nibble), so each packed sign bit expands to one
// nibble instead of one byte: a 128-byte shared-memory row holds 256
// elements, and the tensor core multiplies 4-bit operands at twice its int8
// rate.  Every scale factor is 2^0 (ue8m0 127), every product is +1 or -1,
// and every partial sum is an integer of magnitude at most the padded K
// (<= 2^20, checked by the host), which fp32 holds exactly; the epilogue
// reads the fp32 accumulator as that integer.  Pad positions (bits past K
// and zero-filled words) are +1 in both operands and are subtracted as in
// the int8 kernel.
//
// Roles (sm_100a, one persistent CTA per SM; Cfg below gives the warp counts:
// 11 unpack warps for single CTAs, 8 in a CTA pair):
//  * warp 0     : TMA producer, packed tiles of 128 A rows and the CTA's W
//                 rows x 8 words (256 elements of K, 32-byte swizzle) into a
//                 ring.
//  * warps 2 .. : unpack, one thread per packed row (128 + the W rows).  Each
//                 word becomes 16 bytes: word j of the result is
//                 ((w << (3 - j)) & 0x88888888) | 0x22222222, i.e. nibble i
//                 holds element 4i + j -- a fixed permutation of the word's
//                 32 elements shared by both operands.  One shift and one
//                 LOP3 per 8 elements.  Chunk q of row r is stored at
//                 (q ^ (r & 7)) * 16 (the K-major 128B-swizzled layout).
//  * warp 1     : allocates all 512 TMEM columns (accumulator 0 at column 0,
//                 accumulator 1 at 256, the scale factors at 480..511); one
//                 thread issues 4 tcgen05.mma (M = 128, N = bn, K = 64) per
//                 stage.
//  * last 4     : epilogue: TMEM -> registers -> the fused output modes of
//                 the int8 kernel; dense int32 / fp32 outputs leave as 32 x 32
//                 blocks through swizzled shared memory and TMA tensor stores.
//                 They also fill the scale-factor columns once before the
//                 first MMA.
// Every mbarrier wait is bounded (about 1 s) as in gemm_tc.cuh.
#pragma once

#include "gemm_tc.cuh"

namespace bnn {
namespace f4 {
constexpr int BM = 128;                     // A rows per CTA = TMEM lanes
constexpr int BN_MAX = 224;                 // accumulator columns per tile (bn: a multiple of 32, <= BN_MAX)
constexpr int BKE = 256;                    // elements of K per stage
constexpr int BKW = BKE / 32;               // 8 packed words
constexpr int UMMA_K = 64;                  // e2m1 elements (32 bytes) per tcgen05.mma
constexpr int ROW_BYTES = BKE / 2;          // 128: one unpacked row of a stage
constexpr int P_ROW = BKW * 4;              // 32 bytes of a packed row per stage
constexpr int P_A_BYTES = BM * P_ROW;       // 4 KiB
constexpr int U_A_BYTES = BM * ROW_BYTES;   // 16 KiB
constexpr int EPI_WARPS = 4;
constexpr int WARP_PRODUCER = 0, WARP_MMA = 1, WARP_UNPACK0 = 2;
constexpr int TMEM_COLS = 512;
constexpr int ACC_STRIDE = 256;             // accumulator b starts at column 256 b
constexpr int SF_COL = 480;                 // 32 columns of unit scale factors
constexpr int SFA_COL = SF_COL, SFB_COL = SF_COL + 16;
constexpr uint32_t SF_ONE = 0x7F7F7F7Fu;    // four ue8m0 bytes of 2^0
constexpr int MAX_PSTAGES = 8;
// Output staging for the TMA stores: per epilogue warp one 32 x 32 block of
// int32 and one of fp32 (4 KiB each, 128B-swizzled rows of 32 values).
constexpr int OUT_BLOCK = 32 * 32 * 4;
constexpr int OUT_BYTES = EPI_WARPS * 2 * OUT_BLOCK;
// Per-tile column parameters, one copy shared by the epilogue warps, double
// buffered across tiles: float4 {alpha, gamma, beta, -} and int2 {c1, len2}.
constexpr int COLP_BYTES = 2 * BN_MAX * (16 + 8);
static_assert(ACC_STRIDE + BN_MAX <= SF_COL, "accumulators overlap the scale factors");
static_assert(U_A_BYTES % 1024 == 0 && OUT_BLOCK % 1024 == 0, "swizzled tiles need 1024-byte alignment");
// Named barrier of the epilogue warps (id 0 is __syncthreads).
constexpr int EPI_BAR = 1;
// Bits per code in the plane-code mode: a code c = 0..3 is the e2m1 nibble
// c, the exact value c / 2 (0, 0.5, 1.0, 1.5); the epilogue scales by 4.
constexpr int MAX_F4_PLANES = 2;
// Largest padded K: partial sums stay integers of magnitude <= 2^20, exact
// in fp32 and in the epilogue's float-to-int conversion (valid below 2^22).
constexpr int64_t MAX_KP = int64_t(1) << 20;

// Geometry of one CTA.  Single: the CTA owns a 128 x bn tile.  Pair
// (cta_group::2, a cluster of two CTAs on two SMs): the pair owns a 256 x bn
// tile; each CTA holds its 128 A rows and half of the bn W rows in its
// shared memory and its 128 x bn accumulator in its tensor memory, and the
// even CTA issues the MMAs for both.  Per multiply-add the pair moves
// (128 + bn / 2) instead of (128 + bn) rows through each SM's shared memory.
template <bool PAIR, int MODE = TC_BINARY>
struct Cfg {
    static constexpr int CTAS = PAIR ? 2 : 1;
    static constexpr int BN_CTA_MAX = BN_MAX / CTAS;            // W rows per CTA
    // K atoms (128-byte swizzle atoms, 256 elements) per stage.  CTA pairs
    // of +1/-1 rows take two: each hand-off between the unpack warps and the
    // MMA issuer then covers 512 elements of K (8 MMAs), half as many
    // hand-offs per product; the smaller per-CTA W tile leaves the room.
    static constexpr int KATOMS = (PAIR && MODE != TC_PLANE_CODES) ? 2 : 1;
    static constexpr int S_BKE = BKE * KATOMS;                  // elements of K per stage
    static constexpr int S_BKW = BKW * KATOMS;                  // packed words per row per stage
    static constexpr int S_PROW = P_ROW * KATOMS;               // packed bytes per row per stage
    static constexpr int S_UA = U_A_BYTES * KATOMS;             // unpacked A bytes per stage: [atom][row][128 B]
    static constexpr int USTAGES = PAIR ? (KATOMS == 2 ? 2 : 4) : 3;   // unpacked ring
    static constexpr int U_B_BYTES = BN_CTA_MAX * ROW_BYTES * KATOMS;
    static constexpr int U_STAGE = S_UA + U_B_BYTES;
    // Plane-code mode: every code row brings up to MAX_F4_PLANES packed planes.
    static constexpr int P_STAGE = (BM + BN_CTA_MAX) * S_PROW * (MODE == TC_PLANE_CODES ? MAX_F4_PLANES : 1);
    static constexpr int UNPACK_WARPS = (BM + BN_CTA_MAX + 31) / 32;   // 11 single, 8 pair
    static constexpr int WARP_EPI0 = WARP_UNPACK0 + UNPACK_WARPS;
    static constexpr int THREADS = (WARP_EPI0 + EPI_WARPS) * 32;       // 544 single, 448 pair
    static constexpr int NUM_BARS = 2 * MAX_PSTAGES + 2 * USTAGES + 2 * 2 + 1;
    static constexpr int SMEM_FIXED = USTAGES * U_STAGE + OUT_BYTES + COLP_BYTES + NUM_BARS * 8 + 16 + 1024;
    static constexpr int PSTAGES = (tc::SMEM_LIMIT - SMEM_FIXED) / P_STAGE < MAX_PSTAGES
                                       ? (tc::SMEM_LIMIT - SMEM_FIXED) / P_STAGE
                                       : MAX_PSTAGES;
    static constexpr int SMEM_BYTES = SMEM_FIXED + PSTAGES * P_STAGE;
    static_assert(PSTAGES >= 4, "packed ring too shallow");
    static_assert(SMEM_BYTES <= tc::SMEM_LIMIT, "shared memory");
    static_assert(U_STAGE % 1024 == 0 && S_UA % 1024 == 0 && (BN_CTA_MAX * ROW_BYTES) % 1024 == 0,
                  "unpacked atoms need 1024-byte alignment (128B swizzle)");
    static_assert(P_STAGE % 512 == 0 && (BM * S_PROW) % 512 == 0, "packed stages: 32B / 64B swizzle alignment");
    // Four consecutive epilogue warps have four different (warp & 3): the
    // four TMEM lane quadrants a warp may access.
    static_assert(EPI_WARPS == 4, "one epilogue warp per TMEM lane quadrant");
};
// Block-scaled instruction descriptor: A and B e2m1 (format 1 of kind::mxf4)
// at bits 7-9 and 10-12, both K-major, N >> 3 at bits 17-22, scale format
// ue8m0 (bit 23), M >> 4 at bits 24-28 (M = 128 per CTA of the group);
// scale-factor byte ids 0, K = 64.
__host__ __device__ constexpr uint32_t idesc(int bn, int ctas) {
    return (1u << 7) | (1u << 10) | ((uint32_t)(bn >> 3) << 17) | (1u << 23) | ((uint32_t)((BM * ctas) >> 4) << 24);
}
}  // namespace f4

template <bool PAIR>
__device__ __forceinline__ void mma_mxf4(uint32_t d_tmem, uint64_t adesc, uint64_t bdesc, uint32_t idesc,
                                         uint32_t sfa_tmem, uint32_t sfb_tmem, uint32_t accumulate) {
    if constexpr (PAIR) {
        asm volatile(
            "{\n\t.reg .pred p;\n\t"
            "setp.ne.b32 p, %6, 0;\n\t"
            "tcgen05.mma.cta_group::2.kind::mxf4.block_scale.block32 [%0], %1, %2, %3, [%4], [%5], p;\n\t}" ::"r"(
                d_tmem),
            "l"(adesc), "l"(bdesc), "r"(idesc), "r"(sfa_tmem), "r"(sfb_tmem), "r"(accumulate)
            : "memory");
    } else {
        asm volatile(
            "{\n\t.reg .pred p;\n\t"
            "setp.ne.b32 p, %6, 0;\n\t"
            "tcgen05.mma.cta_group::1.kind::mxf4.block_scale.block32 [%0], %1, %2, %3, [%4], [%5], p;\n\t}" ::"r"(
                d_tmem),
            "l"(adesc), "l"(bdesc), "r"(idesc), "r"(sfa_tmem), "r"(sfb_tmem), "r"(accumulate)
            : "memory");
    }
}

// Arrive on `bar` (the same shared-memory offset in every CTA of `mask`)
// once the MMAs issued so far by this thread are done.
template <bool PAIR>
__device__ __forceinline__ void f4_commit(uint64_t* bar, uint16_t mask) {
    if constexpr (PAIR) {
        asm volatile(
            "tcgen05.commit.cta_group::2.mbarrier::arrive::one.shared::cluster.multicast::cluster.b64 [%0], %1;" ::"r"(
                smem_u32(bar)),
            "h"(mask)
            : "memory");
    } else {
        mma_commit(bar);
    }
}

template <bool PAIR>
__device__ __forceinline__ void f4_tmem_alloc(uint32_t* dst, uint32_t ncols) {
    if constexpr (PAIR) {
        asm volatile("tcgen05.alloc.cta_group::2.sync.aligned.shared::cta.b32 [%0], %1;" ::"r"(smem_u32(dst)),
                     "r"(ncols)
                     : "memory");
        asm volatile("tcgen05.relinquish_alloc_permit.cta_group::2.sync.aligned;" ::: "memory");
    } else {
        tmem_alloc(dst, ncols);
        tmem_relinquish();
    }
}
template <bool PAIR>
__device__ __forceinline__ void f4_tmem_dealloc(uint32_t taddr, uint32_t ncols) {
    if constexpr (PAIR) {
        asm volatile("tcgen05.dealloc.cta_group::2.sync.aligned.b32 %0, %1;" ::"r"(taddr), "r"(ncols) : "memory");
    } else {
        tmem_dealloc(taddr, ncols);
    }
}

__device__ __forceinline__ uint32_t cluster_ctarank() {
    uint32_t r;
    asm volatile("mov.u32 %0, %%cluster_ctarank;" : "=r"(r));
    return r;
}
__device__ __forceinline__ void cluster_sync_all() {
    asm volatile("barrier.cluster.arrive.release.aligned;\n\tbarrier.cluster.wait.acquire.aligned;" ::: "memory");
}
// Arrive on the mbarrier at the same shared-memory offset in CTA `rank` of
// the cluster (release semantics at the default CTA scope: what the arrival
// publishes -- expanded bytes behind a proxy fence, or TMEM reads behind a
// tcgen05 fence -- is consumed by the tensor core, which the waiting thread
// orders after its wait with tcgen05.fence::after_thread_sync).
__device__ __forceinline__ void mbar_arrive_remote(uint64_t* bar, uint32_t rank) {
    asm volatile(
        "{\n\t.reg .b32 ra;\n\t"
        "mapa.shared::cluster.u32 ra, %0, %1;\n\t"
        "mbarrier.arrive.shared::cluster.b64 _, [ra];\n\t}" ::"r"(smem_u32(bar)),
        "r"(rank)
        : "memory");
}

// Registers -> TMEM for one warp: the same 32-bit value in 32 consecutive
// columns of the warp's 32 lanes, then tcgen05.wait::st.
__device__ __forceinline__ void tmem_fill32(uint32_t taddr, uint32_t v) {
    asm volatile(
        "tcgen05.st.sync.aligned.32x32b.x32.b32 [%0], "
        "{%1, %1, %1, %1, %1, %1, %1, %1, %1, %1, %1, %1, %1, %1, %1, %1, "
        "%1, %1, %1, %1, %1, %1, %1, %1, %1, %1, %1, %1, %1, %1, %1, %1};\n\t"
        "tcgen05.wait::st.sync.aligned;" ::"r"(taddr),
        "r"(v)
        : "memory");
}

// Shared -> global tensor store of one box (bulk-group completion), and the
// waits on this thread's outstanding bulk groups.
__device__ __forceinline__ void tma_store_2d(const CUtensorMap* map, const void* smem_src, int32_t x, int32_t y) {
    asm volatile("cp.async.bulk.tensor.2d.global.shared::cta.bulk_group [%0, {%2, %3}], [%1];" ::"l"(
                     reinterpret_cast<uint64_t>(map)),
                 "r"(smem_u32(smem_src)), "r"(x), "r"(y)
                 : "memory");
}
__device__ __forceinline__ void bulk_commit() { asm volatile("cp.async.bulk.commit_group;" ::: "memory"); }
// Wait until at most N of this thread's bulk groups still read shared memory.
template <int N>
__device__ __forceinline__ void bulk_wait_read() {
    asm volatile("cp.async.bulk.wait_group.read %0;" ::"n"(N) : "memory");
}
__device__ __forceinline__ void bulk_wait_all() { asm volatile("cp.async.bulk.wait_group 0;" ::: "memory"); }
__device__ __forceinline__ void named_bar_sync(int id, int threads) {
    asm volatile("bar.sync %0, %1;" ::"r"(id), "r"(threads) : "memory");
}

// 32 sign bits -> 32 e2m1 values (bit 0 -> +1.0 = 0x2, bit 1 -> -1.0 = 0xA)
// in 16 bytes.  Word j of the result holds element 4i + j in nibble i.
__device__ __forceinline__ uint4 expand_word_e2m1(uint32_t w) {
    constexpr uint32_t sign = 0x88888888u, one = 0x22222222u;
    return make_uint4(((w << 3) & sign) | one, ((w << 2) & sign) | one, ((w << 1) & sign) | one, (w & sign) | one);
}

// Bit planes of unsigned codes (one or two planes: codes 0..3) -> e2m1
// values, 16 bytes per 32 codes, in expand_word_e2m1's element order (word
// j, nibble i = element 4i + j).  The e2m1 nibble c (c = 0..3) is the value
// c / 2 (0, 0.5 subnormal, 1.0, 1.5), so a code's nibble is the code itself:
// plane 0 goes to bit 0 of the nibble, plane 1 to bit 1.  The MMA then sums
// (a / 2)(w / 2), a quarter of the code product, and the epilogue scales the
// fp32 accumulator by 4 (exact).
__device__ __forceinline__ uint4 fold_planes_e2m1(uint32_t p0, uint32_t p1) {
    constexpr uint32_t b0 = 0x11111111u, b1 = 0x22222222u;
    return make_uint4((p0 & b0) | ((p1 << 1) & b1), ((p0 >> 1) & b0) | (p1 & b1),
                      ((p0 >> 2) & b0) | ((p1 >> 1) & b1), ((p0 >> 3) & b0) | ((p1 >> 2) & b1));
}

// fp32 accumulator holding an integer of magnitude < 2^22 -> that integer
// (adding 1.5 * 2^23 puts it in the low mantissa bits).
__device__ __forceinline__ int32_t acc_to_int(uint32_t bits) {
    return __float_as_int(__uint_as_float(bits) + 12582912.0f) - 0x4B400000;
}

// The same for an accumulator that holds the integer / scale (scale a power
// of two; the fused multiply-add is exact).
template <int SCALE>
__device__ __forceinline__ int32_t acc_to_int_scaled(uint32_t bits) {
    if constexpr (SCALE == 1) return acc_to_int(bits);
    else return __float_as_int(fmaf(__uint_as_float(bits), (float)SCALE, 12582912.0f)) - 0x4B400000;
}


// MODE (TcMode of gemm_tc.cuh): TC_BINARY the +1/-1 product; TC_PLANE_CODES
// unsigned codes of one or two bit planes (3-D TMA boxes bring a code row's
// planes together, the unpack folds them into e2m1 code values, pads are
// code 0); TC_BASES +1/-1 binary bases, plane-interleaved so that
// accumulator lane L holds base L mod ja of output row L / ja and column c
// base c mod jw of output column c / jw, combined by the epilogue.
template <bool PAIR, int MODE = TC_BINARY>
__global__ void __launch_bounds__(f4::Cfg<PAIR, MODE>::THREADS, 1)
xnor_gemm_f4_kernel(const __grid_constant__ CUtensorMap tmA, const __grid_constant__ CUtensorMap tmW,
                    const __grid_constant__ CUtensorMap tmCi, const __grid_constant__ CUtensorMap tmCf, int M, int N,
                    int K, int kw, int bn, int tiles_m, int tiles_n, int tma_out, GemmEpilogue ep, TcPlanes pl) {
    using namespace f4;
    using C = Cfg<PAIR, MODE>;
    constexpr int CTAS = C::CTAS, USTAGES = C::USTAGES, PSTAGES = C::PSTAGES, U_STAGE = C::U_STAGE,
                  P_STAGE = C::P_STAGE, UNPACK_WARPS = C::UNPACK_WARPS, WARP_EPI0 = C::WARP_EPI0;
    constexpr int KATOMS = C::KATOMS, S_BKE = C::S_BKE, S_BKW = C::S_BKW, S_PROW = C::S_PROW, S_UA = C::S_UA;
    extern __shared__ uint8_t smem_raw[];
    uint8_t* smem = smem_raw + ((1024u - (smem_u32(smem_raw) & 1023u)) & 1023u);
    uint8_t* uring = smem;                                          // USTAGES x (A 16 KiB | W rows)
    uint8_t* oring = uring + USTAGES * U_STAGE;                     // [EPI_WARPS][int32 | fp32] 32 x 32 blocks
    uint8_t* pring = oring + OUT_BYTES;                             // PSTAGES x (A | W packed)
    float4* colf = reinterpret_cast<float4*>(pring + PSTAGES * P_STAGE);   // [2][BN_MAX]
    int2* colt = reinterpret_cast<int2*>(colf + 2 * BN_MAX);               // [2][BN_MAX]
    uint64_t* bars = reinterpret_cast<uint64_t*>(colt + 2 * BN_MAX);
    uint64_t* pfull = bars;
    uint64_t* pempty = pfull + MAX_PSTAGES;
    uint64_t* ufull = pempty + MAX_PSTAGES;
    uint64_t* uempty = ufull + USTAGES;
    uint64_t* afull = uempty + USTAGES;
    uint64_t* aempty = afull + 2;
    uint64_t* drain = aempty + 2;
    uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(drain + 1);
    volatile int* abort_flag = reinterpret_cast<volatile int*>(tmem_slot + 1);

    const int warp = threadIdx.x >> 5;
    const int lane = threadIdx.x & 31;
    const int nk = (kw + S_BKW - 1) / S_BKW;
    const int tiles = tiles_m * tiles_n;
    // Pair: CTA `rank` of cluster `cid` holds A rows 128 rank .. of the
    // tile's 256 and W rows bn_cta rank .. of its bn; the even CTA leads.
    const uint32_t rank = PAIR ? cluster_ctarank() : 0u;
    const int cid = (int)blockIdx.x / CTAS, ncl = (int)gridDim.x / CTAS;
    const int bn_cta = bn / CTAS;
    // Planes per packed A / W row group (plane codes), output rows / columns
    // per CTA and per tile (bases spend ja lanes on a row, jw columns on a column).
    const int ja = MODE == TC_BINARY ? 1 : pl.ja, jw = MODE == TC_BINARY ? 1 : pl.jw;
    const int rows_cta = MODE == TC_BASES ? BM / ja : BM;
    const int cols_tile = MODE == TC_BASES ? bn / jw : bn;
    const int pa_bytes = MODE == TC_PLANE_CODES ? BM * ja * S_PROW : BM * S_PROW;
    const uint32_t stage_tx =
        MODE == TC_PLANE_CODES ? (uint32_t)(BM * ja + bn_cta * jw) * S_PROW : (uint32_t)(BM + bn_cta) * S_PROW;

    if (threadIdx.x == 0) {
        prefetch_tensormap(&tmA);
        prefetch_tensormap(&tmW);
        if (tma_out & 1) prefetch_tensormap(&tmCi);
        if (tma_out & 2) prefetch_tensormap(&tmCf);
        for (int s = 0; s < PSTAGES; ++s) {
            mbar_init(&pfull[s], 1);
            mbar_init(&pempty[s], UNPACK_WARPS);
        }
        for (int s = 0; s < USTAGES; ++s) {
            mbar_init(&ufull[s], UNPACK_WARPS * CTAS);          // the leader's: every unpack warp of the group
            mbar_init(&uempty[s], 1);
        }
        for (int b = 0; b < 2; ++b) {
            mbar_init(&afull[b], 1);
            mbar_init(&aempty[b], EPI_WARPS * CTAS);            // the leader's: every epilogue warp of the group
        }
        mbar_init(drain, 1);
        *abort_flag = 0;
        fence_mbarrier_init();
    }
    if (warp == WARP_MMA) f4_tmem_alloc<PAIR>(tmem_slot, TMEM_COLS);
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem_base = *tmem_slot;
    // Unit scale factors: each epilogue warp fills its 32 lanes of the 32
    // scale-factor columns, so whatever TMEM layout the MMA reads them in,
    // every factor it finds is 2^0.  In a pair both CTAs fill theirs before
    // the cluster barrier, which also publishes the barrier inits to the peer.
    if (warp >= WARP_EPI0) tmem_fill32(tmem_base + ((uint32_t)(32 * (warp & 3)) << 16) + SF_COL, SF_ONE);
    tc_fence_before();
    if constexpr (PAIR) cluster_sync_all(); else __syncthreads();
    tc_fence_after();
    // Programmatic dependent launch (CTA-pair launches carry the attribute):
    // everything above -- barriers, tensor memory, scale factors -- ran while
    // the previous kernel on the stream may still be finishing.  The reads of
    // memory that kernel may write (the operand tiles, the epilogue's column
    // parameters) and every global store come after griddepcontrol.wait in
    // the producer and epilogue warps below.  All CTAs are resident, so the
    // next launch may be scheduled now: its CTAs take SMs as these exit.
    grid_dependents_launch();

    if (warp == WARP_PRODUCER) {
        // ------------------------------ TMA producer ------------------------------
        if (lane == 0) {
            uint32_t g = 0, issued = 0;
            bool ok = true;
            grid_dependency_wait();
            // TMA coordinates in rows of the operand tensors (code or output
            // rows; the 3-D boxes bring each row's planes along).
            const int rows_w = MODE == TC_BASES ? bn_cta / jw : bn_cta;
            for (int t = cid; ok && t < tiles; t += ncl) {
                const int m0 = (t / tiles_n) * (rows_cta * CTAS) + rows_cta * (int)rank;
                const int n0 = (t % tiles_n) * cols_tile + rows_w * (int)rank;
                for (int ks = 0; ks < nk; ++ks, ++g) {
                    const uint32_t s = g % (uint32_t)PSTAGES;
                    if (g >= (uint32_t)PSTAGES && !tc_wait(&pempty[s], ((g / PSTAGES) - 1) & 1, abort_flag)) {
                        ok = false;
                        break;
                    }
                    uint8_t* dst = pring + s * P_STAGE;
                    mbar_arrive_expect_tx(&pfull[s], stage_tx);
                    if constexpr (MODE == TC_BINARY) {
                        tma_load_2d(dst, &tmA, ks * S_BKW, m0, &pfull[s]);
                        tma_load_2d(dst + pa_bytes, &tmW, ks * S_BKW, n0, &pfull[s]);
                    } else {
                        tma_load_3d(dst, &tmA, ks * S_BKW, 0, m0, &pfull[s]);
                        tma_load_3d(dst + pa_bytes, &tmW, ks * S_BKW, 0, n0, &pfull[s]);
                    }
                    ++issued;
                }
            }
            for (uint32_t q = issued > (uint32_t)PSTAGES ? issued - PSTAGES : 0; q < issued; ++q)
                if (!mbar_wait_bounded(&pfull[q % PSTAGES], (q / PSTAGES) & 1)) break;
        }
    } else if (warp == WARP_MMA) {
        // ------------------------------ MMA issuer ------------------------------
        // One thread of the leading CTA; its commits arrive on the barrier of
        // every CTA of the group whose shared or tensor memory they free.
        if (lane == 0 && rank == 0) {
            constexpr uint16_t all = PAIR ? 0x3 : 0x1;
            uint32_t g = 0;
            int lt = 0;
            bool ok = true;
            const uint32_t ubase = smem_u32(uring);
            const uint32_t id = idesc(bn, CTAS);
            const uint32_t sfa = tmem_base + SFA_COL, sfb = tmem_base + SFB_COL;
            for (int t = cid; ok && t < tiles; t += ncl, ++lt) {
                const int b = lt & 1;
                if (lt >= 2 && !tc_wait(&aempty[b], ((lt >> 1) - 1) & 1, abort_flag)) break;
                tc_fence_after();
                const uint32_t d_tmem = tmem_base + (uint32_t)(b * ACC_STRIDE);
                for (int ks = 0; ks < nk; ++ks, ++g) {
                    const uint32_t s = g % USTAGES;
                    if (!tc_wait(&ufull[s], (g / USTAGES) & 1, abort_flag)) {
                        ok = false;
                        break;
                    }
                    tc_fence_after();
                    const uint32_t a_addr = ubase + s * U_STAGE;
                    const uint32_t b_addr = a_addr + S_UA;
                    #pragma unroll
                    for (int kk = 0; kk < S_BKE / UMMA_K; ++kk) {
                        // 32 bytes (64 elements) per K step inside a swizzle atom;
                        // atom kk / 4 of A (B) sits BM (BN_CTA_MAX) rows of 128 B on.
                        const uint32_t ka = (uint32_t)(kk >> 2) * (BM * ROW_BYTES) + (uint32_t)(kk & 3) * 32;
                        const uint32_t kb = (uint32_t)(kk >> 2) * (C::BN_CTA_MAX * ROW_BYTES) + (uint32_t)(kk & 3) * 32;
                        mma_mxf4<PAIR>(d_tmem, umma_desc_sw128(a_addr + ka), umma_desc_sw128(b_addr + kb), id, sfa, sfb,
                                       (ks | kk) != 0 ? 1u : 0u);
                    }
                    f4_commit<PAIR>(&uempty[s], all);
                }
                if (ok) f4_commit<PAIR>(&afull[b], all);
            }
            f4_commit<PAIR>(drain, 0x1);
            mbar_wait_bounded(drain, 0);
        }
        __syncwarp();
    } else if (warp < WARP_EPI0) {
        // ------------------------------ unpack warps ------------------------------
        // Thread u expands packed row u of the stage (A rows 0..127, then the
        // CTA's W rows) into 128 bytes.  Rows are 32 bytes apart in the packed
        // stage, written by the TMA with the 32-byte swizzle: half h of row u
        // sits at 16 * (h ^ ((u >> 2) & 1)), so the eight lanes of a 16-byte
        // load phase hit distinct banks, while the words keep their order for
        // the conflict-free swizzled stores below.
        const int u = threadIdx.x - WARP_UNPACK0 * 32;
        const bool is_a = u < BM;
        const int r = is_a ? u : u - BM;
        const bool active = is_a || r < bn_cta;
        const int sw = r & 7;
        const int hsw = 16 * ((u >> 2) & 1);
        // The stages of all of this CTA's tiles form one sequence; the packed
        // words of stage g + 1 are loaded as soon as stage g is stored, so when
        // the MMAs free the next unpacked buffer the warp only expands.
        const int my_tiles = cid < tiles ? (tiles - 1 - cid) / ncl + 1 : 0;
        const uint32_t total = (uint32_t)my_tiles * (uint32_t)nk;
        uint4 lo = make_uint4(0u, 0u, 0u, 0u), hi = lo;              // words 0..3 and 4..7 of the row
        uint4 lo1 = lo, hi1 = lo;                                     // plane codes: the second plane;
                                                                      // two K atoms: words 8..15
        // Plane codes: the row's planes are consecutive 32-byte slots, from
        // slot s0 on (each slot's halves swizzled by its own index).
        const int nplanes = MODE == TC_PLANE_CODES ? (is_a ? ja : jw) : 1;
        const int s0 = MODE == TC_PLANE_CODES ? (is_a ? r * ja : BM * ja + r * jw) : u;
        auto load_packed = [&](uint32_t gg) -> bool {
            const uint32_t ps = gg % (uint32_t)PSTAGES;
            if (!__all_sync(0xffffffffu, tc_wait(&pfull[ps], (gg / PSTAGES) & 1, abort_flag))) return false;
            if (active) {
                const uint8_t* src = pring + ps * P_STAGE + s0 * S_PROW;
                if constexpr (KATOMS == 2) {
                    // 64-byte rows, written with the 64-byte swizzle: 16-byte
                    // chunk c of slot s0 sits at (c ^ ((s0 >> 1) & 3)) * 16.
                    const int x = (s0 >> 1) & 3;
                    lo = *reinterpret_cast<const uint4*>(src + ((0 ^ x) << 4));
                    hi = *reinterpret_cast<const uint4*>(src + ((1 ^ x) << 4));
                    lo1 = *reinterpret_cast<const uint4*>(src + ((2 ^ x) << 4));
                    hi1 = *reinterpret_cast<const uint4*>(src + ((3 ^ x) << 4));
                } else {
                    const int h0 = MODE == TC_PLANE_CODES ? 16 * ((s0 >> 2) & 1) : hsw;
                    lo = *reinterpret_cast<const uint4*>(src + h0);
                    hi = *reinterpret_cast<const uint4*>(src + (h0 ^ 16));
                    if (MODE == TC_PLANE_CODES && nplanes > 1) {
                        const int h1 = 16 * (((s0 + 1) >> 2) & 1);
                        lo1 = *reinterpret_cast<const uint4*>(src + S_PROW + h1);
                        hi1 = *reinterpret_cast<const uint4*>(src + S_PROW + (h1 ^ 16));
                    }
                }
            }
            return true;
        };
        bool ok = total == 0 || load_packed(0);
        for (uint32_t g = 0; ok && g < total; ++g) {
            const uint32_t ps = g % (uint32_t)PSTAGES, us = g % USTAGES;
            if (!__all_sync(0xffffffffu, g < USTAGES || tc_wait(&uempty[us], ((g / USTAGES) - 1) & 1, abort_flag)))
                break;
            if (active) {
                // Chunk q of the row at (q ^ (r & 7)) * 16: the eight lanes of a
                // store phase (eight consecutive rows) hit distinct banks.
                uint8_t* row = uring + us * U_STAGE + (is_a ? 0 : S_UA) + r * ROW_BYTES;
                if constexpr (KATOMS == 2) {
                    // Words 8..15 go to the second K atom, BM (or BN_CTA_MAX) rows on.
                    uint8_t* row2 = row + (is_a ? BM : C::BN_CTA_MAX) * ROW_BYTES;
                    *reinterpret_cast<uint4*>(row2 + ((0 ^ sw) << 4)) = expand_word_e2m1(lo1.x);
                    *reinterpret_cast<uint4*>(row2 + ((1 ^ sw) << 4)) = expand_word_e2m1(lo1.y);
                    *reinterpret_cast<uint4*>(row2 + ((2 ^ sw) << 4)) = expand_word_e2m1(lo1.z);
                    *reinterpret_cast<uint4*>(row2 + ((3 ^ sw) << 4)) = expand_word_e2m1(lo1.w);
                    *reinterpret_cast<uint4*>(row2 + ((4 ^ sw) << 4)) = expand_word_e2m1(hi1.x);
                    *reinterpret_cast<uint4*>(row2 + ((5 ^ sw) << 4)) = expand_word_e2m1(hi1.y);
                    *reinterpret_cast<uint4*>(row2 + ((6 ^ sw) << 4)) = expand_word_e2m1(hi1.z);
                    *reinterpret_cast<uint4*>(row2 + ((7 ^ sw) << 4)) = expand_word_e2m1(hi1.w);
                }
                if constexpr (MODE == TC_PLANE_CODES) {
                    *reinterpret_cast<uint4*>(row + ((0 ^ sw) << 4)) = fold_planes_e2m1(lo.x, lo1.x);
                    *reinterpret_cast<uint4*>(row + ((1 ^ sw) << 4)) = fold_planes_e2m1(lo.y, lo1.y);
                    *reinterpret_cast<uint4*>(row + ((2 ^ sw) << 4)) = fold_planes_e2m1(lo.z, lo1.z);
                    *reinterpret_cast<uint4*>(row + ((3 ^ sw) << 4)) = fold_planes_e2m1(lo.w, lo1.w);
                    *reinterpret_cast<uint4*>(row + ((4 ^ sw) << 4)) = fold_planes_e2m1(hi.x, hi1.x);
                    *reinterpret_cast<uint4*>(row + ((5 ^ sw) << 4)) = fold_planes_e2m1(hi.y, hi1.y);
                    *reinterpret_cast<uint4*>(row + ((6 ^ sw) << 4)) = fold_planes_e2m1(hi.z, hi1.z);
                    *reinterpret_cast<uint4*>(row + ((7 ^ sw) << 4)) = fold_planes_e2m1(hi.w, hi1.w);
                } else {
                    *reinterpret_cast<uint4*>(row + ((0 ^ sw) << 4)) = expand_word_e2m1(lo.x);
                    *reinterpret_cast<uint4*>(row + ((1 ^ sw) << 4)) = expand_word_e2m1(lo.y);
                    *reinterpret_cast<uint4*>(row + ((2 ^ sw) << 4)) = expand_word_e2m1(lo.z);
                    *reinterpret_cast<uint4*>(row + ((3 ^ sw) << 4)) = expand_word_e2m1(lo.w);
                    *reinterpret_cast<uint4*>(row + ((4 ^ sw) << 4)) = expand_word_e2m1(hi.x);
                    *reinterpret_cast<uint4*>(row + ((5 ^ sw) << 4)) = expand_word_e2m1(hi.y);
                    *reinterpret_cast<uint4*>(row + ((6 ^ sw) << 4)) = expand_word_e2m1(hi.z);
                    *reinterpret_cast<uint4*>(row + ((7 ^ sw) << 4)) = expand_word_e2m1(hi.w);
                }
            }
            if (g + 1 < total) ok = load_packed(g + 1);
            // One proxy fence orders this thread's reads of the packed stage
            // before its next TMA refill and its expanded bytes before the
            // tensor core's reads; then the warp releases the one and hands
            // the other to the MMA issuer (in the leading CTA).
            fence_proxy_async_shared();
            __syncwarp();
            if (lane == 0) {
                mbar_arrive(&pempty[ps]);
                if (rank == 0) mbar_arrive(&ufull[us]);
                else mbar_arrive_remote(&ufull[us], 0);
            }
        }
    } else if constexpr (MODE != TC_BASES) {
        // ------------------------------ epilogue warps ------------------------------
        // Per tile the four warps stage the tile's column parameters in the
        // shared copy of this tile's parity (alpha/gamma/beta and the
        // threshold test as one unsigned range check on the integer
        // accumulator), meet at a named barrier, then each thread turns its
        // row's bn accumulators (fp32 integers) into int32 s, alpha * s, the
        // affine output or the folded-BatchNorm sign bits.  Dense outputs go
        // out as 32 x 32 blocks: the warp writes a block into its staging
        // buffer (row = lane, 16-byte chunk q at (q ^ (lane & 7)) * 16, the
        // TMA's 128-byte swizzle, so no bank conflicts) and lane 0 stores it
        // with one TMA tensor store, which writes whole lines and clips the
        // block at M and N.  Outputs whose pointer or stride does not suit a
        // tensor map are stored directly.  The barrier is reached the same
        // number of times by every warp, also after a failed wait (the warp
        // then skips the work), so it cannot hang.
        grid_dependency_wait();
        const int quad = warp & 3;                                    // TMEM lanes 32*quad .. 32*quad + 31
        const int ew = warp - WARP_EPI0;                              // 0..3
        uint8_t* obuf_i = oring + ew * 2 * OUT_BLOCK;                 // this warp's int32 block
        uint8_t* obuf_f = obuf_i + OUT_BLOCK;                         // and fp32 block
        const bool tma_i = (tma_out & 1) != 0 && ep.c_i32 != nullptr;
        const bool tma_f = (tma_out & 2) != 0 && ep.c_f32 != nullptr;
        const int kp = nk * S_BKE;                                    // padded K: acc = kp - 2 * popcount
        // +1/-1: each pad position adds (+1)(+1); plane codes: pads are code 0.
        const int pad = MODE == TC_PLANE_CODES ? 0 : kp - K;
        const float padf = (float)pad;
        // Plane codes: the accumulator holds a quarter of the code product.
        constexpr int ACC_SCALE = MODE == TC_PLANE_CODES ? 4 : 1;
        const bool affine = ep.gamma != nullptr;
        const int chunks = bn / 32;
        const uint32_t sw = (uint32_t)(lane & 7);
        bool ok = true;
        int lt = 0;
        for (int t = cid; t < tiles; t += ncl, ++lt) {
            const int b = lt & 1;
            const int m0 = (t / tiles_n) * (BM * CTAS) + BM * (int)rank, n0 = (t % tiles_n) * bn;
            float4* cf = colf + b * BN_MAX;
            int2* ct = colt + b * BN_MAX;
            // Every warp finished tile lt - 2 (the last reader of this copy)
            // before it reached the barrier of tile lt - 1.
            for (int i = 32 * ew + lane; i < bn; i += 32 * EPI_WARPS) {
                const int n = n0 + i;
                float4 f = make_float4(0.f, 1.f, 0.f, 0.f);
                int2 th = make_int2(0, 0);                            // len2 = 0: bit never set
                if (n < N) {
                    if (ep.alpha != nullptr) f.x = __ldg(ep.alpha + n);
                    if (affine) { f.y = __ldg(ep.gamma + n); f.z = __ldg(ep.beta + n); }
                    if (ep.c_bits != nullptr) {
                        // bit = (unsigned)(c1 - acc) < 2 len for the interval
                        // [lo, lo + len) of popcounts d = (kp - acc) / 2 that set
                        // the bit (mode 0: d > T; mode 1: d < T; else none).
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
                cf[i] = f;
                ct[i] = th;
            }
            named_bar_sync(EPI_BAR, EPI_WARPS * 32);
            ok = ok && __all_sync(0xffffffffu, tc_wait(&afull[b], (lt >> 1) & 1, abort_flag));
            if (!ok) continue;
            tc_fence_after();
            const int mq = m0 + 32 * quad;                            // first row of this warp's quadrant
            const int m = mq + lane;
            #pragma unroll 1
            for (int c = 0; c < chunks; ++c) {
                uint32_t r[32];
                tmem_ld32_sync(tmem_base + ((uint32_t)(32 * quad) << 16) + (uint32_t)(b * ACC_STRIDE + 32 * c), r);
                if (c == chunks - 1) {
                    // Whole accumulator read: hand it back to the MMA issuer.
                    tc_fence_before();
                    __syncwarp();
                    if (lane == 0) {
                        if (rank == 0) mbar_arrive(&aempty[b]);
                        else mbar_arrive_remote(&aempty[b], 0);
                    }
                }
                const int nb = n0 + 32 * c;
                if (nb >= N) {
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
                        word |= ((uint32_t)(q.x - acc_to_int_scaled<ACC_SCALE>(r[j])) < (uint32_t)q.y ? 1u : 0u) << j;
                    }
                    if (m < M && nb / 32 < ep.bits_words) ep.c_bits[(int64_t)m * ep.ldb + nb / 32] = word;
                }
                if (ep.c_i32 != nullptr && tma_i) {
                    // The block's previous store must have read the buffer
                    // (the other output's store may still be reading its own).
                    if (lane == 0) { if (tma_f) bulk_wait_read<1>(); else bulk_wait_read<0>(); }
                    __syncwarp();
                    uint8_t* rowp = obuf_i + lane * 128;
                    #pragma unroll
                    for (int q = 0; q < 8; ++q)
                        *reinterpret_cast<int4*>(rowp + (((uint32_t)q ^ sw) << 4)) =
                            make_int4(acc_to_int_scaled<ACC_SCALE>(r[4 * q]) - pad,
                                      acc_to_int_scaled<ACC_SCALE>(r[4 * q + 1]) - pad,
                                      acc_to_int_scaled<ACC_SCALE>(r[4 * q + 2]) - pad,
                                      acc_to_int_scaled<ACC_SCALE>(r[4 * q + 3]) - pad);
                    fence_proxy_async_shared();
                    __syncwarp();
                    if (lane == 0) {
                        tma_store_2d(&tmCi, obuf_i, nb, mq);
                        bulk_commit();
                    }
                } else if (m < M && ep.c_i32 != nullptr) {
                    int32_t* dst = ep.c_i32 + (int64_t)m * ep.ldc + nb;
                    const bool vec = full_chunk && ((reinterpret_cast<uintptr_t>(dst) & 15) == 0);
                    #pragma unroll
                    for (int j = 0; j < 32; j += 4) {
                        const int4 o = make_int4(acc_to_int_scaled<ACC_SCALE>(r[j]) - pad,
                                                 acc_to_int_scaled<ACC_SCALE>(r[j + 1]) - pad,
                                                 acc_to_int_scaled<ACC_SCALE>(r[j + 2]) - pad,
                                                 acc_to_int_scaled<ACC_SCALE>(r[j + 3]) - pad);
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
                if (ep.c_f32 != nullptr && (tma_f || m < M)) {
                    // ACC_SCALE * acc - pad is an integer below 2^22: exact
                    // in fp32, so alpha times it is alpha * (float)s.
                    if (tma_f) {
                        if (lane == 0) { if (tma_i) bulk_wait_read<1>(); else bulk_wait_read<0>(); }
                        __syncwarp();
                    }
                    float* dst = ep.c_f32 + (int64_t)m * ep.ldf + nb;
                    const bool vec = full_chunk && ((reinterpret_cast<uintptr_t>(dst) & 15) == 0);
                    #pragma unroll
                    for (int q = 0; q < 8; ++q) {
                        float y[4];
                        #pragma unroll
                        for (int k = 0; k < 4; ++k) {
                            const float4 f = cf[32 * c + 4 * q + k];
                            float v = f.x * fmaf(__uint_as_float(r[4 * q + k]), (float)ACC_SCALE, -padf);
                            if (affine) v = fmaf(f.y, v, f.z);
                            y[k] = v;
                        }
                        if (tma_f) {
                            *reinterpret_cast<float4*>(obuf_f + lane * 128 + (((uint32_t)q ^ sw) << 4)) =
                                make_float4(y[0], y[1], y[2], y[3]);
                        } else if (vec) {
                            *reinterpret_cast<float4*>(dst + 4 * q) = make_float4(y[0], y[1], y[2], y[3]);
                        } else {
                            #pragma unroll
                            for (int k = 0; k < 4; ++k)
                                if (nb + 4 * q + k < N) dst[4 * q + k] = y[k];
                        }
                    }
                    if (tma_f) {
                        fence_proxy_async_shared();
                        __syncwarp();
                        if (lane == 0) {
                            tma_store_2d(&tmCf, obuf_f, nb, mq);
                            bulk_commit();
                        }
                    }
                }
            }
            if (ep.c_bits != nullptr && (t % tiles_n) == tiles_n - 1 && m < M) {
                for (int64_t wd = (int64_t)(n0 + bn) / 32; wd < ep.bits_words; ++wd)
                    ep.c_bits[(int64_t)m * ep.ldb + wd] = 0u;
            }
        }
        // The tensor stores must have finished reading shared memory (and
        // be complete) before the CTA exits.
        if (lane == 0) bulk_wait_all();
        __syncwarp();
    } else {
        // ------------------------- epilogue warps, bases mode -------------------------
        // Accumulator lane L holds base j = L mod ja of output row L / ja of
        // this CTA; column c holds base i = c mod jw of output column c / jw.
        // bases_combine_chunk forms each output from its ja x jw accumulators
        // (ja and jw are powers of two up to 8; one instance per pair).
        // Padded bases have beta_j = 0 or alpha_i[n] = 0 and add exactly 0.
        // The per-tile alpha of every accumulator column sits in the shared
        // double-buffered copy, behind the same named barrier as the other modes.
        grid_dependency_wait();
        const int quad = warp & 3;
        const int ew = warp - WARP_EPI0;
        const int kp = nk * S_BKE;
        const int pad = kp - K;
        const int L = 32 * quad + lane;
        const int jl = L & (ja - 1);
        const float bj = jl < pl.j_real ? __ldg(pl.beta + jl) : 0.0f;
        const int outs_per_chunk = 32 / jw;
        const int chunks = bn / 32;
        const int shape = log2_pow2(ja) * 4 + log2_pow2(jw);
        // 16-byte vector stores where Y's rows keep that alignment.
        const bool vec = ((reinterpret_cast<uintptr_t>(pl.y) | ((uintptr_t)pl.ldy * 4u)) & 15u) == 0;
        bool ok = true;
        int lt = 0;
        for (int t = cid; t < tiles; t += ncl, ++lt) {
            const int b = lt & 1;
            const int m0 = (t / tiles_n) * (rows_cta * CTAS) + rows_cta * (int)rank, n0 = (t % tiles_n) * cols_tile;
            float* ca = reinterpret_cast<float*>(colf + b * BN_MAX);   // alpha of each accumulator column
            for (int i = 32 * ew + lane; i < bn; i += 32 * EPI_WARPS) {
                const int n = n0 + i / jw, ib = i & (jw - 1);
                ca[i] = (n < N && ib < pl.i_real) ? __ldg(pl.alpha + (int64_t)ib * pl.lda_alpha + n) : 0.0f;
            }
            named_bar_sync(EPI_BAR, EPI_WARPS * 32);
            ok = ok && __all_sync(0xffffffffu, tc_wait(&afull[b], (lt >> 1) & 1, abort_flag));
            if (!ok) continue;
            tc_fence_after();
            const int m = m0 + L / ja;
            #pragma unroll 1
            for (int c = 0; c < chunks; ++c) {
                uint32_t r[32];
                tmem_ld32_sync(tmem_base + ((uint32_t)(32 * quad) << 16) + (uint32_t)(b * ACC_STRIDE + 32 * c), r);
                if (c == chunks - 1) {
                    tc_fence_before();
                    __syncwarp();
                    if (lane == 0) {
                        if (rank == 0) mbar_arrive(&aempty[b]);
                        else mbar_arrive_remote(&aempty[b], 0);
                    }
                }
                const int nb = n0 + c * outs_per_chunk;
                if (nb >= N) continue;                                // uniform across the warp
                const float* cc = ca + 32 * c;
                float* yrow = m < M ? pl.y + (int64_t)m * pl.ldy : nullptr;
                bases_combine<false>(shape, r, cc, pad, bj, jl, yrow, nb, N, vec);
            }
        }
    }

    // ------------------------------ teardown ------------------------------
    // In a pair the leader's MMAs read the peer's shared and tensor memory
    // and its commits arrive on the peer's barriers: neither CTA leaves (or
    // frees its tensor memory) before both are done.
    tc_fence_before();
    if constexpr (PAIR) cluster_sync_all(); else __syncthreads();
    if (warp == WARP_MMA) {
        tc_fence_after();
        f4_tmem_dealloc<PAIR>(tmem_base, TMEM_COLS);
    }
}

}  // namespace bnn
