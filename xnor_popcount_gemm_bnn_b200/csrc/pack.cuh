// Sign-and-pack kernels: real tensors -> packed sign bits (+ per-row alpha).
//
// sign(): "Extreme Quantization: Binary, Ternary & 1-bit LLMs", Notation and
// XNOR-Net eq. (4).  Encoding and packing: "First Principles: Why Binary Ops
// Can Be Exponentially Faster", section 1 (bit 0 = +1, bit 1 = -1, pad = +1).
// alpha = (1/K) sum_k |w_k|: "Extreme Quantization ...", eq. (1).
//
// All three kernels are bound by reading the real input from HBM (4 bytes
// in, 1/8 byte out per fp32 element); they use 16-byte vector loads,
// coalesced across the warp, with several loads in flight per lane.
#pragma once

#include "common.cuh"

namespace bnn {

// One warp per row.  A lane loads E = 16/sizeof(T) consecutive elements per
// 16-byte vector; a warp-wide load covers 32*E elements = E words.  Lane l's
// E sign bits land at bit E*(l % G) of word l / G (G = 32/E lanes per word);
// an OR-butterfly over those G lanes assembles the word.
//
// RS: a per-column threshold beta (fp32 [K]), bit = (x < beta_k), i.e.
// sign(x - beta_k) (RSign, "State of the Art Survey (2016 -> 2026)", ReActNet
// row); columns past K use -inf, so their bits stay 0 (+1).  Without RS the
// threshold is 0 (the Notation sign) and beta is not read.
template <typename T, int U, bool RS>
__global__ void __launch_bounds__(256)
pack_sign_rows_kernel(const T* __restrict__ x, int64_t rows, int64_t K, int64_t ld_x,
                      uint32_t* __restrict__ packed, int64_t ldp, float* __restrict__ alpha_out,
                      int64_t kw, bool vec_ok, const float* __restrict__ beta) {
    constexpr int E = 16 / (int)sizeof(T);
    constexpr int G = 32 / E;
    constexpr int CH = 32 * E;  // elements per warp chunk
    const int lane = threadIdx.x & 31;
    const int64_t row = (int64_t)blockIdx.x * (blockDim.x >> 5) + (threadIdx.x >> 5);
    if (row >= rows) return;
    const T* xr = x + row * ld_x;
    uint32_t* pr = packed + row * ldp;
    const int64_t nchunks = (kw * 32 + CH - 1) / CH;
    double asum = 0.0;

    for (int64_t c0 = 0; c0 < nchunks; c0 += U) {
        float v[U][E];
        #pragma unroll
        for (int u = 0; u < U; ++u) {
            const int64_t base = (c0 + u) * CH + (int64_t)lane * E;
            if (vec_ok && base + E <= K) {
                uint4 q = ldg_stream_v4(xr + base);
                const T* e = reinterpret_cast<const T*>(&q);
                #pragma unroll
                for (int i = 0; i < E; ++i) v[u][i] = to_float(e[i]);
            } else {
                #pragma unroll
                for (int i = 0; i < E; ++i)
                    v[u][i] = (base + i < K) ? to_float(xr[base + i]) : 0.0f;
            }
        }
        #pragma unroll
        for (int u = 0; u < U; ++u) {
            const int64_t chunk = c0 + u;
            if (chunk >= nchunks) break;
            uint32_t bits = 0;
            if constexpr (!RS) {
                #pragma unroll
                for (int i = 0; i < E; ++i) {
                    bits |= neg_bit(v[u][i]) << i;
                    asum += fabs((double)v[u][i]);  // elements past K were loaded as 0
                }
            } else {
                const int64_t base = chunk * CH + (int64_t)lane * E;
                #pragma unroll
                for (int i = 0; i < E; ++i) {
                    const float b = base + i < K ? __ldg(beta + base + i) : -INFINITY;
                    bits |= (v[u][i] < b ? 1u : 0u) << i;
                    asum += fabs((double)v[u][i]);
                }
            }
            bits <<= E * (lane % G);
            #pragma unroll
            for (int off = 1; off < G; off <<= 1) bits |= __shfl_xor_sync(0xffffffffu, bits, off);
            const int64_t wi = chunk * E + lane / G;
            if ((lane % G) == 0 && wi < kw) pr[wi] = bits;
        }
    }
    if (alpha_out != nullptr) {
        #pragma unroll
        for (int off = 16; off >= 1; off >>= 1) asum += __shfl_xor_sync(0xffffffffu, asum, off);
        if (lane == 0) alpha_out[row] = (float)(asum / (double)K);
    }
}

// Raw bits of one element, and element p of a 16-byte vector as float.
__device__ __forceinline__ uint32_t raw_bits(float v) { return __float_as_uint(v); }
__device__ __forceinline__ uint32_t raw_bits(__nv_bfloat16 v) { return (uint32_t)__bfloat16_as_ushort(v); }
template <typename T>
__device__ __forceinline__ float vec_elem(const uint32_t (&w)[4], int p) {
    if constexpr (sizeof(T) == 4) {
        return __uint_as_float(w[p]);
    } else {
        const uint32_t x = w[p >> 1];
        return __uint_as_float((p & 1) ? (x & 0xFFFF0000u) : (x << 16));   // bf16 -> fp32 is exact
    }
}

// NCHW real activations -> per-pixel channel words [n, h, w, cw].
// A warp task is word j of 8*E consecutive pixels of one image (E = pixels
// per 16-byte vector: 8 bf16, 4 fp32).  Lane (g, q) = (lane / 4, lane % 4)
// owns pixels [g*E, g*E + E) of the task and channels 32j + 8q .. + 7: eight
// 16-byte loads, issued together by one asm statement so that all eight are
// in flight before any is used.  For one channel the 32 lanes read 4 rows x
// 128 contiguous bytes, so every load instruction is 4 full lines.  Each lane
// sets bits 8q .. 8q+7 of its E pixels' words; two shuffles OR the four
// quarters together, and lane q stores the pixels p = q (mod 4).
// RS: per-channel threshold beta (fp32 [c]), bit = (x < beta_c) (RSign, as in
// pack_sign_rows_kernel); channels past c use -inf.
template <typename T, bool RS>
__global__ void __launch_bounds__(256)
pack_sign_nchw_kernel(const T* __restrict__ x, int64_t n, int64_t c, int64_t hw, int64_t cw,
                      uint32_t* __restrict__ out, bool vec_ok, const float* __restrict__ beta) {
    constexpr int E = 16 / (int)sizeof(T);
    constexpr int PX = 8 * E;                     // pixels per task
    const int lane = threadIdx.x & 31;
    const int g = lane >> 2, q = lane & 3;
    const int64_t groups = (hw + PX - 1) / PX;
    const int64_t task = ((int64_t)blockIdx.x * blockDim.x + threadIdx.x) >> 5;
    if (task >= n * groups * cw) return;          // whole warps leave together
    const int64_t j = task % cw;
    const int64_t gi = (task / cw) % groups;
    const int64_t b = task / (cw * groups);
    const int64_t p0 = gi * PX + g * E;           // this lane's first pixel
    const int np = (int)(hw - p0 <= 0 ? 0 : (hw - p0 < E ? hw - p0 : E));
    const int64_t ch0 = 32 * j + 8 * q;           // this lane's first channel
    const int nc = (int)(c - ch0 <= 0 ? 0 : (c - ch0 < 8 ? c - ch0 : 8));
    const T* src = x + ((b * c + (nc > 0 ? ch0 : 0)) * hw + (np > 0 ? p0 : 0));
    uint32_t v[8][4];                             // raw 16-byte vectors, one per channel
    if (vec_ok && np == E && nc == 8) {
        const size_t rs = (size_t)hw * sizeof(T);     // one channel row, in bytes
        const char* a = reinterpret_cast<const char*>(src);
        asm volatile(
            "ld.global.nc.v4.u32 {%0, %1, %2, %3}, [%32];\n\t"
            "ld.global.nc.v4.u32 {%4, %5, %6, %7}, [%33];\n\t"
            "ld.global.nc.v4.u32 {%8, %9, %10, %11}, [%34];\n\t"
            "ld.global.nc.v4.u32 {%12, %13, %14, %15}, [%35];\n\t"
            "ld.global.nc.v4.u32 {%16, %17, %18, %19}, [%36];\n\t"
            "ld.global.nc.v4.u32 {%20, %21, %22, %23}, [%37];\n\t"
            "ld.global.nc.v4.u32 {%24, %25, %26, %27}, [%38];\n\t"
            "ld.global.nc.v4.u32 {%28, %29, %30, %31}, [%39];"
            : "=r"(v[0][0]), "=r"(v[0][1]), "=r"(v[0][2]), "=r"(v[0][3]),
              "=r"(v[1][0]), "=r"(v[1][1]), "=r"(v[1][2]), "=r"(v[1][3]),
              "=r"(v[2][0]), "=r"(v[2][1]), "=r"(v[2][2]), "=r"(v[2][3]),
              "=r"(v[3][0]), "=r"(v[3][1]), "=r"(v[3][2]), "=r"(v[3][3]),
              "=r"(v[4][0]), "=r"(v[4][1]), "=r"(v[4][2]), "=r"(v[4][3]),
              "=r"(v[5][0]), "=r"(v[5][1]), "=r"(v[5][2]), "=r"(v[5][3]),
              "=r"(v[6][0]), "=r"(v[6][1]), "=r"(v[6][2]), "=r"(v[6][3]),
              "=r"(v[7][0]), "=r"(v[7][1]), "=r"(v[7][2]), "=r"(v[7][3])
            : "l"(a), "l"(a + rs), "l"(a + 2 * rs), "l"(a + 3 * rs), "l"(a + 4 * rs), "l"(a + 5 * rs),
              "l"(a + 6 * rs), "l"(a + 7 * rs));
    } else {
        // Ragged pixels or channels: element loads, zeros (+1) elsewhere.
        #pragma unroll
        for (int i = 0; i < 8; ++i) {
            #pragma unroll
            for (int k = 0; k < 4; ++k) {
                uint32_t w = 0;
                #pragma unroll
                for (int t = 0; t < E / 4; ++t) {
                    const int pp = k * (E / 4) + t;
                    const uint32_t raw = (i < nc && pp < np) ? raw_bits(src[(int64_t)i * hw + pp]) : 0u;
                    w |= raw << (32 / (E / 4) * t);
                }
                v[i][k] = w;
            }
        }
    }
    uint32_t bits[E];
    if constexpr (RS) {
        float th[8];
        #pragma unroll
        for (int i = 0; i < 8; ++i) th[i] = i < nc ? __ldg(beta + ch0 + i) : -INFINITY;
        #pragma unroll
        for (int p = 0; p < E; ++p) {
            uint32_t w = 0;
            #pragma unroll
            for (int i = 0; i < 8; ++i) w |= (vec_elem<T>(v[i], p) < th[i] ? 1u : 0u) << i;
            bits[p] = w << (8 * q);
        }
    } else {
        #pragma unroll
        for (int p = 0; p < E; ++p) {
            uint32_t w = 0;
            #pragma unroll
            for (int i = 0; i < 8; ++i) w |= neg_bit(vec_elem<T>(v[i], p)) << i;
            bits[p] = w << (8 * q);
        }
    }
    #pragma unroll
    for (int p = 0; p < E; ++p) {
        bits[p] |= __shfl_xor_sync(0xffffffffu, bits[p], 1);
        bits[p] |= __shfl_xor_sync(0xffffffffu, bits[p], 2);
    }
    #pragma unroll
    for (int p = 0; p < E; ++p)
        if ((p & 3) == q && p < np) out[(b * hw + p0 + p) * cw + j] = bits[p];
}

// The same NCHW -> per-pixel channel words, streamed by TMA.  A tile is 32
// channel rows x 128 bytes of pixels (64 bf16 or 32 fp32) of one image:
// channels 32j .. 32j+31 of pixels [t*P, t*P + P), 4 KiB.  Every warp is its
// own pipeline over the tiles gw, gw + W, gw + 2W, ... (W = warps in the
// grid) with STAGES tiles in flight in its own part of shared memory, so with
// one 512-thread block per SM the whole activation tensor of a ResNet layer
// is requested at once and HBM streams without waves or register limits.
// Lane l reads 4 bytes of each of the 32 rows (pixels 2l, 2l+1 for bf16, l
// for fp32; a warp reads one 128-byte row per load, no bank conflicts) and
// builds the whole 32-bit channel word of its pixels itself.  Rows past c
// belong to the next image (or lie past the tensor, zero-filled) and are
// masked; pixels past hw are zero-filled and not stored.
// RS: per-channel threshold beta (fp32 [c]), bit = (x < beta_c).
namespace nchw_tma {
constexpr int WARPS = 16;
constexpr int THREADS = 32 * WARPS;
constexpr int STAGES = 3;
constexpr int TILE_BYTES = 32 * 128;
constexpr int SMEM_BYTES = WARPS * STAGES * TILE_BYTES + WARPS * STAGES * 8;
}  // namespace nchw_tma

template <typename T, bool RS>
__global__ void __launch_bounds__(nchw_tma::THREADS, 1)
pack_sign_nchw_tma_kernel(const __grid_constant__ CUtensorMap map, int64_t n, int64_t c, int64_t hw, int64_t cw,
                          int64_t tiles_per_plane, uint32_t* __restrict__ out, const float* __restrict__ beta) {
    using namespace nchw_tma;
    constexpr int P = 128 / (int)sizeof(T);       // pixels per tile
    constexpr int PPL = P / 32;                   // pixels per lane
    extern __shared__ __align__(1024) uint8_t smem[];
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    uint8_t* tiles = smem + warp * STAGES * TILE_BYTES;
    uint64_t* bars = reinterpret_cast<uint64_t*>(smem + WARPS * STAGES * TILE_BYTES) + warp * STAGES;
    const int64_t total = n * cw * tiles_per_plane;
    const int64_t gw = (int64_t)blockIdx.x * WARPS + warp;
    const int64_t nw = (int64_t)gridDim.x * WARPS;
    if (lane == 0) {
        prefetch_tensormap(&map);
        #pragma unroll
        for (int s = 0; s < STAGES; ++s) mbar_init(&bars[s], 1);
        fence_mbarrier_init();
    }
    __syncwarp();
    auto issue = [&](int64_t u, int s) {
        const int64_t t = u % tiles_per_plane, bj = u / tiles_per_plane;
        const int64_t j = bj % cw, b = bj / cw;
        mbar_arrive_expect_tx(&bars[s], TILE_BYTES);
        tma_load_2d(tiles + s * TILE_BYTES, &map, (int32_t)(t * P), (int32_t)(b * c + 32 * j), &bars[s]);
    };
    if (lane == 0) {
        #pragma unroll
        for (int s = 0; s < STAGES; ++s)
            if (gw + s * nw < total) issue(gw + s * nw, s);
    }
    const int64_t mine = gw < total ? (total - gw + nw - 1) / nw : 0;   // tiles of this warp
    int k = 0;
    for (int64_t u = gw; u < total; u += nw, ++k) {
        const int s = k % STAGES;
        const bool ok = mbar_wait_bounded(&bars[s], (uint32_t)((k / STAGES) & 1));
        if (!__all_sync(0xffffffffu, ok)) {
            // gave up (the error flag is set): wait, bounded, for the tiles
            // still in flight into this warp's stages before leaving
            const int64_t issued = min(mine, (int64_t)k + STAGES);
            for (int64_t i = k + 1; i < issued; ++i) mbar_wait_bounded(&bars[i % STAGES], (uint32_t)((i / STAGES) & 1));
            break;
        }
        const int64_t t = u % tiles_per_plane, bj = u / tiles_per_plane;
        const int64_t j = bj % cw, b = bj / cw;
        const int64_t cvalid = c - 32 * j;
        const uint32_t mask = cvalid >= 32 ? 0xffffffffu : ((1u << cvalid) - 1u);
        const uint8_t* tile = tiles + s * TILE_BYTES;
        uint32_t wd[PPL];
        // Each row costs one compare that writes a mask register and one LOP3
        // that keeps that row's bit: x < th as an ordered compare, so -0.0 and
        // NaN give 0 and negative subnormals give 1, as in the other packs.
        if constexpr (sizeof(T) == 2) {
            // Two pixels per lane as one bf16x2.  For a bf16 x and an fp32
            // threshold b, x < b exactly when x < (b rounded up to bf16), so
            // the compare runs in bf16x2 with no loss.  Rows 0..15 gather in
            // acc0 (pixel 2l in bits 0..15, pixel 2l+1 in bits 16..31), rows
            // 16..31 in acc1.
            uint32_t th_lane = 0u;
            if constexpr (RS) {
                const __nv_bfloat16 tb =
                    __float2bfloat16_ru((32 * j + lane < c) ? __ldg(beta + 32 * j + lane) : 0.0f);
                const uint32_t h = (uint32_t)__bfloat16_as_ushort(tb);
                th_lane = h | (h << 16);
            }
            uint32_t acc0 = 0u, acc1 = 0u;
            #pragma unroll
            for (int r = 0; r < 32; ++r) {
                const uint32_t raw = *reinterpret_cast<const uint32_t*>(tile + r * 128 + lane * 4);
                uint32_t tb2 = 0u;
                if constexpr (RS) tb2 = __shfl_sync(0xffffffffu, th_lane, r);
                const uint32_t m = __hlt2_mask(*reinterpret_cast<const __nv_bfloat162*>(&raw),
                                               *reinterpret_cast<const __nv_bfloat162*>(&tb2));
                if (r < 16) acc0 |= m & (0x00010001u << r);
                else        acc1 |= m & (0x00010001u << (r - 16));
            }
            wd[0] = (acc0 & 0xFFFFu) | (acc1 << 16);
            wd[PPL - 1] = (acc0 >> 16) | (acc1 & 0xFFFF0000u);
        } else {
            float th_lane = 0.0f;
            if constexpr (RS) th_lane = (32 * j + lane < c) ? __ldg(beta + 32 * j + lane) : 0.0f;
            uint32_t acc = 0u;
            #pragma unroll
            for (int r = 0; r < 32; ++r) {
                const float v = *reinterpret_cast<const float*>(tile + r * 128 + lane * 4);
                float th = 0.0f;
                if constexpr (RS) th = __shfl_sync(0xffffffffu, th_lane, r);
                uint32_t m;
                asm("set.lt.u32.f32 %0, %1, %2;" : "=r"(m) : "f"(v), "f"(th));
                acc |= m & (1u << r);
            }
            wd[0] = acc;
        }
        // the stage's bytes were read through the generic proxy; order those
        // reads before the next TMA write into the same bytes
        fence_proxy_async_shared();
        __syncwarp();
        if (lane == 0 && u + STAGES * nw < total) issue(u + STAGES * nw, s);
        #pragma unroll
        for (int q = 0; q < PPL; ++q) {
            const int64_t p = t * P + lane * PPL + q;
            if (p < hw) out[(b * hw + p) * cw + j] = wd[q] & mask;
        }
    }
}

// OIHW 3x3 filters -> packed rows in (kh, kw, c) order, one warp per output
// channel; lane = channel within a 32-channel word.  alpha over the 9*cin
// true weights (eq. (1): one scale per filter).
template <typename T>
__global__ void __launch_bounds__(256)
pack_conv3x3_weights_kernel(const T* __restrict__ w, int64_t cout, int64_t cin,
                            uint32_t* __restrict__ packed, int64_t ldp, float* __restrict__ alpha_out) {
    const int lane = threadIdx.x & 31;
    const int64_t co = (int64_t)blockIdx.x * (blockDim.x >> 5) + (threadIdx.x >> 5);
    if (co >= cout) return;
    const int64_t cw = (cin + 31) / 32;
    const int64_t words = 9 * cw;
    const int64_t ldk = (words + 3) / 4 * 4;
    uint32_t* pr = packed + co * ldp;
    double asum = 0.0;
    for (int t = 0; t < 9; ++t) {
        for (int64_t j = 0; j < cw; ++j) {
            const int64_t ch = 32 * j + lane;
            const float v = (ch < cin) ? to_float(w[(co * cin + ch) * 9 + t]) : 0.0f;
            asum += fabs((double)v);
            const uint32_t word = __ballot_sync(0xffffffffu, v < 0.0f);
            if (lane == 0) pr[t * cw + j] = word;
        }
    }
    for (int64_t wi = words + lane; wi < ldk; wi += 32) pr[wi] = 0u;
    if (alpha_out != nullptr) {
        #pragma unroll
        for (int off = 16; off >= 1; off >>= 1) asum += __shfl_xor_sync(0xffffffffu, asum, off);
        if (lane == 0) alpha_out[co] = (float)(asum / (double)(9 * cin));
    }
}

// Unsigned k-bit codes -> bit planes ("State of the Art Survey (2016 ->
// 2026)", classic CNN BNN table, DoReFa-Net: low-bit weights and activations
// multiplied by bit-convolution).  codes: uint8 [rows, ld_codes], only the low
// `bits` bits of each byte are used.  planes: plane p of row r is the packed
// row r * bits + p (stride ldw words), bit j of word w = bit p of code
// 32 w + j; elements past K and words up to kw are zero.  One warp per row; a
// lane takes 16 consecutive codes (one 16-byte load when aligned), each plane's
// 16 bits are gathered 4 codes at a time with a multiply (bits at 0, 8, 16, 24
// land on 28..31 without carries), and two neighbouring lanes form a word.
__global__ void __launch_bounds__(256)
pack_bit_planes_kernel(const uint8_t* __restrict__ codes, int64_t rows, int64_t K, int64_t ldc, int bits,
                       uint32_t* __restrict__ planes, int64_t ldw, int64_t kw, bool vec) {
    const int lane = threadIdx.x & 31;
    const int64_t row = (int64_t)blockIdx.x * (blockDim.x >> 5) + (threadIdx.x >> 5);
    if (row >= rows) return;                                  // warp-uniform
    const uint8_t* src = codes + row * ldc;
    uint32_t* dst = planes + row * bits * ldw;
    for (int64_t w0 = 0; w0 < kw; w0 += 16) {                 // 16 words (512 codes) per warp pass
        const int64_t e0 = 32 * w0 + 16 * (int64_t)lane;      // this lane's first code
        uint32_t x[4];
        if (vec && e0 + 16 <= K) {
            const uint4 q = *reinterpret_cast<const uint4*>(src + e0);
            x[0] = q.x; x[1] = q.y; x[2] = q.z; x[3] = q.w;
        } else {
            #pragma unroll
            for (int q = 0; q < 4; ++q) {
                uint32_t v = 0;
                #pragma unroll
                for (int i = 0; i < 4; ++i) {
                    const int64_t e = e0 + 4 * q + i;
                    if (e < K) v |= (uint32_t)src[e] << (8 * i);
                }
                x[q] = v;
            }
        }
        const int64_t wd = w0 + (lane >> 1);
        for (int p = 0; p < bits; ++p) {
            uint32_t b16 = 0;
            #pragma unroll
            for (int q = 0; q < 4; ++q) {
                const uint32_t y = (x[q] >> p) & 0x01010101u;
                b16 |= ((y * 0x10204080u) >> 28) << (4 * q);
            }
            uint32_t word = b16 << (16 * (lane & 1));
            word |= __shfl_xor_sync(0xffffffffu, word, 1);
            if ((lane & 1) == 0 && wd < kw) dst[(int64_t)p * ldw + wd] = word;
        }
    }
}

}  // namespace bnn
