// Binary 3x3 convolution on the tensor cores: the implicit GEMM of conv.cuh
// (M = output pixels, N = filters, K = 9 taps x C channels; "Extreme
// Quantization: Binary, Ternary & 1-bit LLMs", eq. (4), (6), eq. (1) per
// filter) computed with tcgen05.mma kind::i8 on +1/-1 bytes.
//
// Every product is +1 or -1 and the int32 accumulation is exact, so the
// result equals 9*C - 2 * popcount over the gathered words.  Positions that
// are padding in both operands -- channels past C inside a tap's words and
// the words that round the row up to whole 128-element stages -- hold 0 bits
// (+1) on both sides; each adds (+1)(+1), and the epilogue subtracts their
// count KPAD - 9*C.  A tap outside the image is the all-zero word in the
// activation only (+1 times the filter bit): a real term, as in conv.cuh.
//
// Design (sm_100a, one persistent CTA per SM, 9 warps):
//  * The filters (N <= 256 rows of 9*CW words) are expanded once per CTA into
//    shared memory in the K-major 128B-swizzled layout and stay resident.
//  * warps 1-4: gather + unpack.  Thread r owns output pixel r of the tile:
//    it loads its 9 taps x CW words from the packed NHWC activations (L2
//    resident; padded taps read 0), then writes NS stages of 128 signed bytes
//    into the tile's A buffer (two buffers: the next tile is gathered while
//    the tensor cores work on this one).
//  * warp 0: allocates TMEM (two 128 x N int32 accumulators) and one thread
//    issues NS x 4 tcgen05.mma (M = 128, N, K = 32) per tile.
//  * warps 5-8: epilogue.  Thread = output pixel, 32 filters per tcgen05.ld;
//    the NCHW stores of a warp are 32 consecutive pixels of one filter plane.
//  * Every wait is bounded; on time-out the CTA records BNN_ERR_DEVICE_TIMEOUT,
//    the roles stop, the MMAs drain and TMEM is freed before exit.
#pragma once

#include "common.cuh"
#include "conv.cuh"      // ConvEpilogue
#include "gemm_tc.cuh"   // tcgen05 helpers, expand_word_pm1, umma_desc_sw128
#include "gemm_f4.cuh"   // e2m1 expansion, kind::mxf4 MMA, unit scale factors

namespace bnn {
namespace ctc {
constexpr int BM = 128;                    // output pixels per tile (TMEM lanes)
constexpr int MAX_N = 256;
constexpr int GATHER_WARPS = 4;
constexpr int EPI_WARPS = 4;
constexpr int WARP_MMA = 0, WARP_GATHER0 = 1, WARP_EPI0 = WARP_GATHER0 + GATHER_WARPS;
constexpr int THREADS = (WARP_EPI0 + EPI_WARPS) * 32;   // 288
constexpr int STAGE_A_BYTES = BM * 128;    // 16 KiB per 128-element stage
}  // namespace ctc

// Shared-memory bytes for CW words per tap and N (a multiple of 16) filter rows.
__host__ __device__ constexpr int conv_tc_stages(int cw) { return (9 * cw + 3) / 4; }
__host__ __device__ inline int conv_tc_smem_bytes(int cw, int n) {
    const int ns = conv_tc_stages(cw);
    return 2 * ns * ctc::STAGE_A_BYTES + ns * n * 128 + 16 * 8 + 16 + 1024;
}

// Writes 32 sign bits of a packed word as 32 signed bytes (+1 / -1) into two
// 16-byte chunks (2q, 2q+1) of a 128-byte swizzled row (expand_word_pm1's
// element order, shared by both operands).
__device__ __forceinline__ void expand_word_sw128(uint8_t* row, int q, int sw, uint32_t w) {
    uint4 c0, c1;
    expand_word_pm1(w, c0, c1);
    *reinterpret_cast<uint4*>(row + (((2 * q) ^ sw) << 4)) = c0;
    *reinterpret_cast<uint4*>(row + (((2 * q + 1) ^ sw) << 4)) = c1;
}

template <int CW>
__global__ void __launch_bounds__(ctc::THREADS, 1)
xnor_conv3x3_tc_kernel(const uint32_t* __restrict__ X, int n, int c, int h, int w,
                       const uint32_t* __restrict__ Wp, int64_t ldw, int cout, int n_mma, uint32_t idesc,
                       int stride, int pad, int oh, int ow, ConvEpilogue ep) {
    using namespace ctc;
    constexpr int KW = 9 * CW;                  // real words per row
    constexpr int NS = conv_tc_stages(CW);      // 128-element stages
    constexpr int KWP = 4 * NS;                 // words per row incl. pad words
    extern __shared__ uint8_t smem_raw[];
    uint8_t* smem = smem_raw + ((1024u - (smem_u32(smem_raw) & 1023u)) & 1023u);
    uint8_t* abuf = smem;                                          // 2 x NS x 16 KiB
    uint8_t* bsm = smem + 2 * NS * STAGE_A_BYTES;                  // NS x n_mma x 128 B
    uint64_t* bars = reinterpret_cast<uint64_t*>(bsm + NS * n_mma * 128);
    uint64_t* afill = bars;            // [2] A buffer gathered (count: gather warps)
    uint64_t* accfull = afill + 2;     // [2] MMAs of the tile done (tcgen05.commit)
    uint64_t* accempty = accfull + 2;  // [2] accumulator drained (count: epilogue warps)
    uint64_t* drain = accempty + 2;
    uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(drain + 1);
    volatile int* abort_flag = reinterpret_cast<volatile int*>(tmem_slot + 1);

    const int warp = threadIdx.x >> 5;
    const int lane = threadIdx.x & 31;
    const int64_t plane = (int64_t)oh * ow;
    const int64_t npix = (int64_t)n * plane;
    const int tiles = (int)((npix + BM - 1) / BM);
    // Two accumulators at 32-column aligned offsets; the allocation is a power of 2.
    const int acc_stride = (n_mma + 31) / 32 * 32;
    const uint32_t tmem_cols = acc_stride <= 64 ? 128u : (acc_stride <= 128 ? 256u : 512u);

    if (threadIdx.x == 0) {
        for (int b = 0; b < 2; ++b) {
            mbar_init(&afill[b], GATHER_WARPS);
            mbar_init(&accfull[b], 1);
            mbar_init(&accempty[b], EPI_WARPS);
        }
        mbar_init(drain, 1);
        *abort_flag = 0;
        fence_mbarrier_init();
    }
    if (warp == WARP_MMA) {
        tmem_alloc(tmem_slot, tmem_cols);
        tmem_relinquish();
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem_base = *tmem_slot;

    if (warp == WARP_MMA) {
        // ------------------------------ MMA issuer ------------------------------
        if (lane == 0) {
            int lt = 0;
            const uint32_t a0 = smem_u32(abuf), b0 = smem_u32(bsm);
            for (int t = blockIdx.x; t < tiles; t += gridDim.x, ++lt) {
                const int b = lt & 1;
                if (!tc_wait(&afill[b], (lt >> 1) & 1, abort_flag)) break;
                if (lt >= 2 && !tc_wait(&accempty[b], ((lt >> 1) - 1) & 1, abort_flag)) break;
                tc_fence_after();
                const uint32_t d_tmem = tmem_base + (uint32_t)(b * acc_stride);
                #pragma unroll
                for (int s = 0; s < NS; ++s) {
                    #pragma unroll
                    for (int kk = 0; kk < 4; ++kk) {
                        const uint64_t ad = umma_desc_sw128(a0 + (b * NS + s) * STAGE_A_BYTES + kk * 32);
                        const uint64_t bd = umma_desc_sw128(b0 + s * n_mma * 128 + kk * 32);
                        asm volatile(
                            "{\n\t.reg .pred p;\n\t"
                            "setp.ne.b32 p, %4, 0;\n\t"
                            "tcgen05.mma.cta_group::1.kind::i8 [%0], %1, %2, %3, p;\n\t}" ::"r"(d_tmem),
                            "l"(ad), "l"(bd), "r"(idesc), "r"((s | kk) != 0 ? 1u : 0u)
                            : "memory");
                    }
                }
                mma_commit(&accfull[b]);
            }
            mma_commit(drain);
            mbar_wait_bounded(drain, 0);       // every MMA done before TMEM is freed
        }
        __syncwarp();
    } else if (warp < WARP_EPI0) {
        // --------------------------- gather + unpack warps ---------------------------
        const int r = threadIdx.x - WARP_GATHER0 * 32;             // tile row 0..127
        const int sw = r & 7;
        // Filters first: rows r (and r + 128) of B, all stages, once per CTA.
        for (int fr = r; fr < n_mma; fr += BM) {
            uint32_t wd[KWP];
            #pragma unroll
            for (int k = 0; k < KWP; ++k) wd[k] = (fr < cout && k < KW) ? __ldg(Wp + (int64_t)fr * ldw + k) : 0u;
            #pragma unroll
            for (int s = 0; s < NS; ++s) {
                uint8_t* row = bsm + s * n_mma * 128 + fr * 128;
                #pragma unroll
                for (int q = 0; q < 4; ++q) expand_word_sw128(row, q, fr & 7, wd[4 * s + q]);
            }
        }
        int lt = 0;
        for (int t = blockIdx.x; t < tiles; t += gridDim.x, ++lt) {
            const int b = lt & 1;
            // The A buffer is free once the MMAs of tile lt - 2 are done.
            const bool ok = lt < 2 || tc_wait(&accfull[b], ((lt >> 1) - 1) & 1, abort_flag);
            if (!__all_sync(0xffffffffu, ok)) break;
            const int64_t q = (int64_t)t * BM + r;
            int64_t bi = 0, oy = 0, ox = 0;
            if (q < npix) {
                bi = q / plane;
                const int64_t rem = q % plane;
                oy = rem / ow;
                ox = rem % ow;
            }
            uint32_t wd[KWP];
            #pragma unroll
            for (int tap = 0; tap < 9; ++tap) {
                const int iy = (int)oy * stride - pad + tap / 3;
                const int ix = (int)ox * stride - pad + tap % 3;
                const bool in = q < npix && iy >= 0 && iy < h && ix >= 0 && ix < w;
                const int64_t off = in ? ((bi * h + iy) * (int64_t)w + ix) * CW : 0;
                #pragma unroll
                for (int j = 0; j < CW; ++j) wd[tap * CW + j] = in ? __ldg(X + off + j) : 0u;
            }
            #pragma unroll
            for (int k = KW; k < KWP; ++k) wd[k] = 0u;
            #pragma unroll
            for (int s = 0; s < NS; ++s) {
                uint8_t* row = abuf + (b * NS + s) * STAGE_A_BYTES + r * 128;
                #pragma unroll
                for (int qq = 0; qq < 4; ++qq) expand_word_sw128(row, qq, sw, wd[4 * s + qq]);
            }
            fence_proxy_async_shared();
            __syncwarp();
            if (lane == 0) mbar_arrive(&afill[b]);
        }
    } else {
        // ------------------------------ epilogue warps ------------------------------
        const int quad = warp & 3;
        const int padc = NS * 128 - 9 * c;           // (+1)(+1) pad positions per output
        int lt = 0;
        for (int t = blockIdx.x; t < tiles; t += gridDim.x, ++lt) {
            const int b = lt & 1;
            if (!__all_sync(0xffffffffu, tc_wait(&accfull[b], (lt >> 1) & 1, abort_flag))) break;
            tc_fence_after();
            const int64_t q = (int64_t)t * BM + 32 * quad + lane;
            const bool valid = q < npix;
            const int64_t obase = valid ? (q / plane) * cout * plane + q % plane : 0;
            for (int c0 = 0; c0 < n_mma; c0 += 32) {
                uint32_t rr[32];
                tmem_ld32_sync(tmem_base + ((uint32_t)(32 * quad) << 16) + (uint32_t)(b * acc_stride + c0), rr);
                if (c0 + 32 >= n_mma) {
                    tc_fence_before();
                    __syncwarp();
                    if (lane == 0) mbar_arrive(&accempty[b]);
                }
                if (!valid) continue;
                #pragma unroll
                for (int j = 0; j < 32; ++j) {
                    const int co = c0 + j;
                    if (co >= cout) break;
                    const int32_t sv = (int32_t)rr[j] - padc;
                    const int64_t o = obase + (int64_t)co * plane;
                    if (ep.mode == BNN_OUT_INT32) {
                        static_cast<int32_t*>(ep.out)[o] = sv;
                    } else {
                        float y = __ldg(ep.alpha + co) * (float)sv;
                        if (ep.mode == BNN_OUT_AFFINE_F32) y = fmaf(__ldg(ep.gamma + co), y, __ldg(ep.beta + co));
                        static_cast<float*>(ep.out)[o] = y;
                    }
                }
            }
        }
    }

    tc_fence_before();
    __syncthreads();
    if (warp == WARP_MMA) {
        tc_fence_after();
        tmem_dealloc(tmem_base, tmem_cols);
    }
}

// ---------------------------------------------------------------------------
// Stride-1 binary 3x3 convolution on the tensor cores with shifted windows.
//
// Index the zero-padded input of every image on a "virtual" line: position
// u = b*Hp*Wp + y*Wp + x with Hp = h + 2*pad, Wp = w + 2*pad.  The output
// pixel (b, oy, ox), placed at u = b*Hp*Wp + oy*Wp + ox, reads tap (dy, dx)
// at u + dy*Wp + dx, so for 128 consecutive positions every tap is the same
// 128-row matrix shifted by a constant number of rows.  Each input position
// is expanded to +1/-1 bytes once, into a buffer of consecutive positions in
// the non-swizzled K-major operand layout (rows 16 B apart inside each 16-byte
// column of K), and the 9 * CW MMAs of a tile take their A operand at a
// different row offset of that buffer.  Positions of the line with oy >= oh or
// ox >= ow are computed and dropped.
//
// The sums are exact: (+1)(+1) for the pad bits of each tap's last word is
// subtracted (9 * (32*CW - C) per output); an out-of-image tap reads the zero
// word (+1), as in conv.cuh.
//
// A CTA owns a contiguous range of 128-position tiles and walks it in
// segments that fit one of two A buffers.  Inside a segment consecutive tiles
// share 2*Wp + 2 halo rows, so a tile expands 128 new rows; the first tile of
// a segment expands its whole window.  A buffer is refilled only after the
// MMAs of the segment that last used it are done (a tcgen05.commit per
// segment).
//
// Warps: 0 = TMEM owner and MMA issuer, 1-4 = expansion (one row per thread),
// 5-20 = epilogue in two groups of eight: group i drains the accumulator of
// tiles k = i (mod 2), i.e. always TMEM buffer i, so one group's stores run
// while the other waits for its MMAs and TMEM load.  Inside a group, two warps
// per TMEM lane quadrant take alternate 16-column slices.  The fp32 NCHW
// output is the largest stream of the kernel.  All waits are bounded as in
// the kernel above.
// ---------------------------------------------------------------------------
namespace ctw {
constexpr int BM = 128;
constexpr int GATHER_WARPS = 4;
constexpr int EPI_WARPS = 16;                            // two groups of 8
constexpr int EPI_GROUP = 8;
constexpr int EPI_COLS = 16;                             // columns per tcgen05.ld slice
constexpr int WARP_MMA = 0, WARP_GATHER0 = 1, WARP_EPI0 = WARP_GATHER0 + GATHER_WARPS;
constexpr int THREADS = (WARP_EPI0 + EPI_WARPS) * 32;   // 672
constexpr int AHEAD = 4;                                 // tiles the expansion may run ahead
constexpr int BAR_BYTES = 192;                           // 15 mbarriers, TMEM slot, abort flag
}  // namespace ctw

struct ConvWindow {
    int n, h, w, pad;
    int Hp, Wp, oh, ow;
    int V;           // n * Hp * Wp virtual positions
    int tiles;       // ceil(V / 128)
    int rb;          // rows per A buffer (multiple of 8)
    int seg_tiles;   // tiles per segment: 128 * seg_tiles + halo <= rb
    int halo;        // 2 * Wp + 2
};

// Operand geometry of the window kernel.  int8 (+1/-1 bytes): an A row is
// 32 bytes per packed word, a filter stage 128 elements.  e2m1 (+1/-1
// nibbles, F4): 16 bytes per word, 256 elements per filter stage.
__host__ __device__ constexpr int conv_tcw_row_bytes(int cw, bool f4) { return cw * (f4 ? 16 : 32); }
__host__ __device__ constexpr int conv_tcw_b_stages(int cw, bool f4) {
    return f4 ? (9 * cw + 7) / 8 : conv_tc_stages(cw);
}
// Shared-memory bytes for CW words per pixel, n_mma filter rows and rb rows
// per A buffer.
__host__ __device__ inline int conv_tcw_smem_bytes(int cw, int n_mma, int rb, bool f4 = false) {
    return 1024 + conv_tcw_b_stages(cw, f4) * n_mma * 128 + 2 * rb * conv_tcw_row_bytes(cw, f4) + 12 * n_mma +
           ctw::BAR_BYTES;
}

// Non-swizzled K-major shared-memory descriptor: rows 16 B apart inside a
// core matrix, 8-row groups sbo bytes apart, the two 16-byte K halves of one
// K = 32 step lbo bytes apart.
__device__ __forceinline__ uint64_t umma_desc_interleave(uint32_t smem_addr, uint32_t lbo, uint32_t sbo) {
    return (uint64_t)((smem_addr >> 4) & 0x3FFFu) | ((uint64_t)((lbo >> 4) & 0x3FFFu) << 16) |
           ((uint64_t)((sbo >> 4) & 0x3FFFu) << 32) | ((uint64_t)1u << 46);
}

// F4: the same kernel on e2m1 operands (tcgen05.mma kind::mxf4 with unit
// block scales, CW even): a pixel's word expands to 16 bytes instead of 32,
// one K = 64 MMA covers two words, and the fp32 accumulators hold exact
// integers (at most 9 * 32 * CW in magnitude).
template <int CW, bool F4 = false>
__global__ void __launch_bounds__(ctw::THREADS, 1)
xnor_conv3x3_tcw_kernel(const uint32_t* __restrict__ X, int c, const uint32_t* __restrict__ Wp_,
                        int64_t ldw, int cout, int n_mma, uint32_t idesc, ConvWindow g, ConvEpilogue ep) {
    using namespace ctw;
    static_assert(!F4 || CW % 2 == 0, "e2m1 MMAs take two words of K");
    constexpr int KW = 9 * CW;
    constexpr int NS = conv_tcw_b_stages(CW, F4);
    constexpr int KWP = (F4 ? 8 : 4) * NS;
    extern __shared__ uint8_t smem_raw[];
    uint8_t* smem = smem_raw + ((1024u - (smem_u32(smem_raw) & 1023u)) & 1023u);
    uint8_t* bsm = smem;                                                   // NS x n_mma x 128 B, SW128
    const int abuf_stride = g.rb * conv_tcw_row_bytes(CW, F4);
    uint8_t* abuf = bsm + NS * n_mma * 128;                                // 2 x abuf_stride
    float* s_alpha = reinterpret_cast<float*>(abuf + 2 * abuf_stride);     // [n_mma]
    float* s_gamma = s_alpha + n_mma;
    float* s_beta = s_gamma + n_mma;
    uint64_t* bars = reinterpret_cast<uint64_t*>(s_beta + n_mma);
    uint64_t* afill = bars;               // [AHEAD] window of the tile expanded (count: gather warps)
    uint64_t* aconsumed = afill + AHEAD;  // [AHEAD] the MMA thread has seen that afill phase
    uint64_t* accfull = aconsumed + AHEAD;  // [2] MMAs of the tile done
    uint64_t* accempty = accfull + 2;  // [2] accumulator read out (count: epilogue warps)
    uint64_t* segfree = accempty + 2;  // [2] MMAs of the last segment in A buffer i done
    uint64_t* drain = segfree + 2;
    uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(drain + 1);
    volatile int* abort_flag = reinterpret_cast<volatile int*>(tmem_slot + 1);

    const int warp = threadIdx.x >> 5;
    const int lane = threadIdx.x & 31;
    const int tb = (int)((int64_t)blockIdx.x * g.tiles / gridDim.x);
    const int te = (int)((int64_t)(blockIdx.x + 1) * g.tiles / gridDim.x);
    const int kt = te - tb;
    const int HpWp = g.Hp * g.Wp;
    const int acc_stride = (n_mma + 31) / 32 * 32;
    // e2m1: 32 columns of unit scale factors after the two accumulators.
    const int used_cols = 2 * acc_stride + (F4 ? 32 : 0);
    const uint32_t tmem_cols = used_cols <= 128 ? 128u : (used_cols <= 256 ? 256u : 512u);
    const uint32_t sf_col = (uint32_t)(2 * acc_stride);

    if (threadIdx.x == 0) {
        for (int b = 0; b < AHEAD; ++b) {
            mbar_init(&afill[b], GATHER_WARPS);
            mbar_init(&aconsumed[b], 1);
        }
        for (int b = 0; b < 2; ++b) {
            mbar_init(&accfull[b], 1);
            mbar_init(&accempty[b], EPI_GROUP);
            mbar_init(&segfree[b], 1);
        }
        mbar_init(drain, 1);
        *abort_flag = 0;
        fence_mbarrier_init();
    }
    if (warp == WARP_MMA) {
        tmem_alloc(tmem_slot, tmem_cols);
        tmem_relinquish();
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem_base = *tmem_slot;
    if constexpr (F4) {
        // The first four epilogue warps (one per TMEM lane quadrant) write
        // the scale factors, all 2^0, before the first MMA.
        if (warp >= WARP_EPI0 && warp < WARP_EPI0 + 4)
            tmem_fill32(tmem_base + ((uint32_t)(32 * (warp & 3)) << 16) + sf_col, f4::SF_ONE);
        tc_fence_before();
        __syncthreads();
        tc_fence_after();
    }
    // Programmatic dependent launch: the set-up above ran while the previous
    // kernel on the stream may still be finishing.  Every read of memory it
    // may write (epilogue parameters, filters, the packed input) and every
    // store come after this wait.  The grid is resident, so the next launch
    // may be scheduled now; its CTAs take SMs as these exit.
    grid_dependents_launch();
    grid_dependency_wait();
    for (int i = threadIdx.x; i < n_mma; i += blockDim.x) {
        const bool real = i < cout && ep.mode != BNN_OUT_INT32;
        s_alpha[i] = real ? __ldg(ep.alpha + i) : 0.0f;
        s_gamma[i] = real && ep.mode == BNN_OUT_AFFINE_F32 ? __ldg(ep.gamma + i) : 0.0f;
        s_beta[i] = real && ep.mode == BNN_OUT_AFFINE_F32 ? __ldg(ep.beta + i) : 0.0f;
    }
    __syncthreads();

    if (warp == WARP_MMA) {
        // ------------------------------ MMA issuer ------------------------------
        if (lane == 0) {
            // Descriptors are built once; per MMA only the start-address field
            // (bits 0-13, in 16-byte units) moves, and every smem address here
            // is below 256 KB, so a 32-bit add on the low word cannot carry
            // into the other fields.  This keeps the issuing thread short: it
            // shares its SM sub-partition with expansion and epilogue warps.
            const uint64_t ad0 = umma_desc_interleave(smem_u32(abuf), (uint32_t)g.rb * 16u, 128u);
            const uint64_t bd0 = umma_desc_sw128(smem_u32(bsm));
            const uint32_t ad_lo = (uint32_t)ad0, ad_hi = (uint32_t)(ad0 >> 32);
            const uint32_t bd_lo = (uint32_t)bd0, bd_hi = (uint32_t)(bd0 >> 32);
            const uint32_t row_dy[3] = {0u, (uint32_t)g.Wp, 2u * (uint32_t)g.Wp};   // tap row shift, in rows
            const uint32_t khalf = 2u * (uint32_t)g.rb;                           // one 32-byte K step, in 16-B units
            const uint32_t bstage = (uint32_t)n_mma * 8u;                          // one B stage, in 16-B units
            for (int k = 0; k < kt; ++k) {
                const int b = k & 1;
                const int seg = k / g.seg_tiles, ks = k - seg * g.seg_tiles;
                if (!tc_wait(&afill[k % AHEAD], (k / AHEAD) & 1, abort_flag)) break;
                mbar_arrive(&aconsumed[k % AHEAD]);
                if (k >= 2 && !tc_wait(&accempty[b], ((k >> 1) - 1) & 1, abort_flag)) break;
                tc_fence_after();
                const uint32_t d_tmem = tmem_base + (uint32_t)(b * acc_stride);
                const uint32_t a_tile = ad_lo + (uint32_t)(((seg & 1) * abuf_stride) >> 4) + (uint32_t)(ks * BM);
                // One K step is 32 bytes of a row: two A planes (khalf apart)
                // and two 16-byte chunks of a filter stage; int8 takes one
                // word per step, e2m1 two.
                constexpr int STEPS = F4 ? CW / 2 : CW;                  // K steps per tap
                #pragma unroll
                for (int tap = 0; tap < 9; ++tap) {
                    const uint32_t a_tap = a_tile + row_dy[tap / 3] + (uint32_t)(tap % 3);
                    #pragma unroll
                    for (int j = 0; j < STEPS; ++j) {
                        const int wk = tap * STEPS + j;
                        const uint64_t ad = ((uint64_t)ad_hi << 32) | (a_tap + (uint32_t)j * khalf);
                        const uint64_t bd = ((uint64_t)bd_hi << 32) |
                                            (bd_lo + (uint32_t)(wk / 4) * bstage + (uint32_t)((wk % 4) * 2));
                        if constexpr (F4) {
                            mma_mxf4<false>(d_tmem, ad, bd, idesc, tmem_base + sf_col, tmem_base + sf_col + 16,
                                            wk != 0 ? 1u : 0u);
                        } else {
                            asm volatile(
                                "{\n\t.reg .pred p;\n\t"
                                "setp.ne.b32 p, %4, 0;\n\t"
                                "tcgen05.mma.cta_group::1.kind::i8 [%0], %1, %2, %3, p;\n\t}" ::"r"(d_tmem),
                                "l"(ad), "l"(bd), "r"(idesc), "r"(wk != 0 ? 1u : 0u)
                                : "memory");
                        }
                    }
                }
                mma_commit(&accfull[b]);
                if (ks == g.seg_tiles - 1 || k == kt - 1) mma_commit(&segfree[seg & 1]);
            }
            mma_commit(drain);
            mbar_wait_bounded(drain, 0);       // every MMA done before TMEM is freed
        }
        __syncwarp();
    } else if (warp < WARP_EPI0) {
        // ------------------------------ expansion warps ------------------------------
        const int r = threadIdx.x - WARP_GATHER0 * 32;                 // 0..127
        for (int fr = r; fr < n_mma; fr += BM) {
            uint32_t wd[KWP];
            #pragma unroll
            for (int k = 0; k < KWP; ++k) wd[k] = (fr < cout && k < KW) ? __ldg(Wp_ + (int64_t)fr * ldw + k) : 0u;
            #pragma unroll
            for (int s = 0; s < NS; ++s) {
                uint8_t* row = bsm + s * n_mma * 128 + fr * 128;
                if constexpr (F4) {
                    #pragma unroll
                    for (int q = 0; q < 8; ++q)
                        *reinterpret_cast<uint4*>(row + ((q ^ (fr & 7)) << 4)) = expand_word_e2m1(wd[8 * s + q]);
                } else {
                    #pragma unroll
                    for (int q = 0; q < 4; ++q) expand_word_sw128(row, q, fr & 7, wd[4 * s + q]);
                }
            }
        }
        for (int k = 0; k < kt; ++k) {
            const int seg = k / g.seg_tiles, ks = k - seg * g.seg_tiles;
            // Inside a segment rows are only appended, so the expansion runs up
            // to AHEAD tiles ahead of the MMAs; a buffer is refilled once the
            // MMAs of the segment that used it before are done.
            const bool ok = ks != 0 || seg < 2 || tc_wait(&segfree[seg & 1], ((seg >> 1) - 1) & 1, abort_flag);
            if (!__all_sync(0xffffffffu, ok)) break;
            const int useg = (tb + seg * g.seg_tiles) * BM;           // position of buffer row 0
            const int row_lo = ks == 0 ? 0 : ks * BM + g.halo;
            const int row_hi = ks * BM + BM + g.halo;
            uint8_t* ab = abuf + (seg & 1) * abuf_stride;
            for (int row = row_lo + r; row < row_hi; row += BM) {
                const int u = useg + row;
                uint32_t wd[CW];
                #pragma unroll
                for (int j = 0; j < CW; ++j) wd[j] = 0u;
                if (u < g.V) {
                    const int bi = u / HpWp;
                    const int rem = u - bi * HpWp;
                    const int yp = rem / g.Wp;
                    const int iy = yp - g.pad, ix = rem - yp * g.Wp - g.pad;
                    if (iy >= 0 && iy < g.h && ix >= 0 && ix < g.w) {
                        const uint32_t* src = X + (((int64_t)bi * g.h + iy) * g.w + ix) * CW;
                        #pragma unroll
                        for (int j = 0; j < CW; ++j) wd[j] = __ldg(src + j);
                    }
                }
                #pragma unroll
                for (int j = 0; j < CW; ++j) {
                    if constexpr (F4) {
                        *reinterpret_cast<uint4*>(ab + j * g.rb * 16 + row * 16) = expand_word_e2m1(wd[j]);
                    } else {
                        uint4 c0, c1;
                        expand_word_pm1(wd[j], c0, c1);
                        *reinterpret_cast<uint4*>(ab + (2 * j) * g.rb * 16 + row * 16) = c0;
                        *reinterpret_cast<uint4*>(ab + (2 * j + 1) * g.rb * 16 + row * 16) = c1;
                    }
                }
            }
            fence_proxy_async_shared();
            // afill[k % AHEAD] is re-armed only after the MMA thread has seen
            // its previous phase (tile k - AHEAD).
            const bool ok2 = k < AHEAD || tc_wait(&aconsumed[k % AHEAD], ((k / AHEAD) - 1) & 1, abort_flag);
            if (!__all_sync(0xffffffffu, ok2)) break;
            __syncwarp();
            if (lane == 0) mbar_arrive(&afill[k % AHEAD]);
        }
    } else {
        // ------------------------------ epilogue warps ------------------------------
        const int e = warp - WARP_EPI0;               // 0..15
        const int grp = e / EPI_GROUP;                // tiles k = grp (mod 2): TMEM buffer grp
        const int quad = warp & 3;                    // TMEM lanes 32*quad .. +31
        const int slice0 = EPI_COLS * ((e % EPI_GROUP) >> 2);   // slices slice0, slice0 + 32, ...
        const int padc = 9 * (32 * CW - c);           // (+1)(+1) pad positions per output
        const int64_t ohow = (int64_t)g.oh * g.ow;
        const int lane_pos = 32 * quad + lane;        // this thread's row of every tile
        for (int k = grp; k < kt; k += 2) {
            const int b = grp;
            if (!__all_sync(0xffffffffu, tc_wait(&accfull[b], (k >> 1) & 1, abort_flag))) break;
            tc_fence_after();
            const int u = (tb + k) * BM + lane_pos;
            const int bi = u / HpWp;
            const int rem = u - bi * HpWp;
            const int oy = rem / g.Wp, ox = rem - (rem / g.Wp) * g.Wp;
            const bool valid = u < g.V && oy < g.oh && ox < g.ow;
            const int64_t obase = valid ? ((int64_t)bi * cout * g.oh + oy) * g.ow + ox : 0;
            bool arrived = false;
            for (int c0 = slice0; c0 < n_mma; c0 += 2 * EPI_COLS) {
                uint32_t rr[EPI_COLS];
                tmem_ld16_sync(tmem_base + ((uint32_t)(32 * quad) << 16) + (uint32_t)(b * acc_stride + c0), rr);
                if (c0 + 2 * EPI_COLS >= n_mma) {
                    tc_fence_before();
                    __syncwarp();
                    if (lane == 0) mbar_arrive(&accempty[b]);
                    arrived = true;
                }
                if (!valid) continue;
                if (F4 && ep.mode == BNN_OUT_INT32) {
                    // fp32 accumulators holding integers (|acc| < 2^22): read
                    // them as the int32 values the int8 path produces.
                    #pragma unroll
                    for (int jj = 0; jj < EPI_COLS; ++jj) rr[jj] = (uint32_t)acc_to_int(rr[jj]);
                }
                if (ep.mode == BNN_OUT_INT32) {
                    int32_t* o = static_cast<int32_t*>(ep.out) + obase;
                    #pragma unroll
                    for (int jj = 0; jj < EPI_COLS; ++jj)
                        if (c0 + jj < cout) o[(int64_t)(c0 + jj) * ohow] = (int32_t)rr[jj] - padc;
                } else {
                    float* o = static_cast<float*>(ep.out) + obase;
                    const bool affine = ep.mode == BNN_OUT_AFFINE_F32;
                    #pragma unroll
                    for (int j4 = 0; j4 < EPI_COLS; j4 += 4) {
                        const float4 a4 = *reinterpret_cast<const float4*>(s_alpha + c0 + j4);
                        const float4 g4 = *reinterpret_cast<const float4*>(s_gamma + c0 + j4);
                        const float4 b4 = *reinterpret_cast<const float4*>(s_beta + c0 + j4);
                        const float av[4] = {a4.x, a4.y, a4.z, a4.w};
                        const float gv[4] = {g4.x, g4.y, g4.z, g4.w};
                        const float bv[4] = {b4.x, b4.y, b4.z, b4.w};
                        #pragma unroll
                        for (int q = 0; q < 4; ++q) {
                            const int co = c0 + j4 + q;
                            // s = acc - pad exactly: an int32 subtraction, or for the
                            // e2m1 accumulators one fp32 subtraction of two integers
                            // below 2^22 (the same float as (float)s).
                            const float sf = F4 ? __uint_as_float(rr[j4 + q]) - (float)padc
                                                : (float)((int32_t)rr[j4 + q] - padc);
                            float y = av[q] * sf;
                            if (affine) y = fmaf(gv[q], y, bv[q]);
                            if (co < cout) o[(int64_t)co * ohow] = y;
                        }
                    }
                }
            }
            if (!arrived) {
                tc_fence_before();
                __syncwarp();
                if (lane == 0) mbar_arrive(&accempty[b]);
            }
        }
    }

    tc_fence_before();
    __syncthreads();
    if (warp == WARP_MMA) {
        tc_fence_after();
        tmem_dealloc(tmem_base, tmem_cols);
    }
}

}  // namespace bnn
