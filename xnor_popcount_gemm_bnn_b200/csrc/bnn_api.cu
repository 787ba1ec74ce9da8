// libbnn.so: the C ABI declared in include/bnn.h.  Host code here only checks
// arguments, encodes TMA descriptors, picks launch shapes and launches on the
// caller's stream; every step of the computation runs in the kernels of
// pack.cuh, gemm_popc.cuh, gemm_tc.cuh, gemm_f4.cuh, gemv.cuh, chain.cuh, bwgemv.cuh, conv.cuh,
// conv_tc.cuh and ternary.cuh.
#include <cudaTypedefs.h>

#include <atomic>
#include <cmath>
#include <climits>
#include <cstdint>
#include <cstring>
#include <algorithm>
#include <mutex>

#include "bnn.h"
#include "chain.cuh"
#include "common.cuh"
#include "conv.cuh"
#include "conv_tc.cuh"
#include "conv1x1.cuh"
#include "gemm_popc.cuh"
#include "gemm_tc.cuh"
#include "gemm_f4.cuh"
#include "gemv.cuh"
#include "hostio.cuh"
#include "bwgemv.cuh"
#include "bwgemv_i8.cuh"
#include "pack.cuh"
#include "probe.cuh"
#include "ternary.cuh"

namespace {

using bnn::packed_ld_words;

inline bool aligned(const void* p, uintptr_t a) { return (reinterpret_cast<uintptr_t>(p) & (a - 1)) == 0; }

inline cudaStream_t as_cuda(bnn_stream_t s) { return reinterpret_cast<cudaStream_t>(s); }

inline bnn_status launch_status() {
    return cudaGetLastError() == cudaSuccess ? BNN_OK : BNN_ERR_CUDA;
}

inline int64_t ceil_div(int64_t a, int64_t b) { return (a + b - 1) / b; }

// Resident CTA-pair count that marks the pair mode of the 4-bit GEMM as unavailable.
constexpr int kNoPairs = 1 << 30;

// cuTensorMapEncodeTiled from the driver, fetched through the runtime so that
// the library does not link libcuda directly.
PFN_cuTensorMapEncodeTiled_v12000 tensor_map_encoder() {
    static PFN_cuTensorMapEncodeTiled_v12000 fn = nullptr;
    static std::once_flag once;
    std::call_once(once, [] {
        void* p = nullptr;
        cudaDriverEntryPointQueryResult q{};
        if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &p, cudaEnableDefault, &q) == cudaSuccess &&
            q == cudaDriverEntryPointSuccess)
            fn = reinterpret_cast<PFN_cuTensorMapEncodeTiled_v12000>(p);
    });
    return fn;
}

// 2-D map over a packed matrix: inner dimension = kw words, outer = rows,
// box 32 words x box_rows rows, 128-byte swizzle, zero fill out of range.
bool encode_packed_map(CUtensorMap* map, const uint32_t* base, int64_t kw, int64_t rows, int64_t ld,
                       int box_rows, int box_words = bnn::gemm::BKW,
                       CUtensorMapSwizzle swizzle = CU_TENSOR_MAP_SWIZZLE_128B) {
    auto enc = tensor_map_encoder();
    if (enc == nullptr) return false;
    cuuint64_t dims[2] = {(cuuint64_t)kw, (cuuint64_t)rows};
    cuuint64_t strides[1] = {(cuuint64_t)ld * 4u};
    cuuint32_t box[2] = {(cuuint32_t)box_words, (cuuint32_t)box_rows};
    cuuint32_t estr[2] = {1, 1};
    CUresult r = enc(map, CU_TENSOR_MAP_DATA_TYPE_UINT32, 2, const_cast<uint32_t*>(base), dims, strides,
                     box, estr, CU_TENSOR_MAP_INTERLEAVE_NONE, swizzle,
                     CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
    return r == CUDA_SUCCESS;
}

// Opt the GEMM kernel into its dynamic shared memory once per device (the
// attribute is per device; doing it once keeps it out of captured graphs).
bool gemm_smem_configured() {
    constexpr int kMaxDevices = 64;
    static std::atomic<int> done[kMaxDevices];
    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess || dev < 0) return false;
    if (dev < kMaxDevices && done[dev].load(std::memory_order_acquire)) return true;
    if (cudaFuncSetAttribute(bnn::xnor_gemm_popc_kernel<bnn::gemm::TN, bnn::gemm::CSA>,
                             cudaFuncAttributeMaxDynamicSharedMemorySize, bnn::gemm::SMEM_BYTES) != cudaSuccess)
        return false;
    if (dev < kMaxDevices) done[dev].store(1, std::memory_order_release);
    return true;
}

// Per-device one-time opt-in to the tensor-core GEMM's shared memory.
bool gemm_tc_smem_configured() {
    constexpr int kMaxDevices = 64;
    static std::atomic<int> done[kMaxDevices];
    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess || dev < 0) return false;
    if (dev < kMaxDevices && done[dev].load(std::memory_order_acquire)) return true;
    if (cudaFuncSetAttribute(bnn::xnor_gemm_tc_kernel<bnn::TC_BINARY>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                             bnn::tc::SMEM_BYTES) != cudaSuccess ||
        cudaFuncSetAttribute(bnn::xnor_gemm_tc_kernel<bnn::TC_PLANE_CODES>,
                             cudaFuncAttributeMaxDynamicSharedMemorySize, bnn::tc::SMEM_LIMIT) != cudaSuccess ||
        cudaFuncSetAttribute(bnn::xnor_gemm_tc_kernel<bnn::TC_BASES>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                             bnn::tc::SMEM_BYTES) != cudaSuccess)
        return false;
    if (dev < kMaxDevices) done[dev].store(1, std::memory_order_release);
    return true;
}

// Per-device one-time opt-in to the 4-bit tensor-core GEMM's shared memory
// (both modes), and the number of CTA pairs that fit on the device at once.
int gemm_f4_pairs_resident() {
    constexpr int kMaxDevices = 64;
    static std::atomic<int> pairs[kMaxDevices];              // 0: not configured yet
    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess || dev < 0) return -1;
    if (dev < kMaxDevices) {
        const int p = pairs[dev].load(std::memory_order_acquire);
        if (p > 0) return p;
    }
    using C1 = bnn::f4::Cfg<false>;
    using C2 = bnn::f4::Cfg<true>;
    if (cudaFuncSetAttribute(bnn::xnor_gemm_f4_kernel<false>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                             C1::SMEM_BYTES) != cudaSuccess ||
        cudaFuncSetAttribute(bnn::xnor_gemm_f4_kernel<true>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                             C2::SMEM_BYTES) != cudaSuccess ||
        cudaFuncSetAttribute(bnn::xnor_gemm_f4_kernel<true, bnn::TC_PLANE_CODES>,
                             cudaFuncAttributeMaxDynamicSharedMemorySize,
                             bnn::f4::Cfg<true, bnn::TC_PLANE_CODES>::SMEM_BYTES) != cudaSuccess ||
        cudaFuncSetAttribute(bnn::xnor_gemm_f4_kernel<true, bnn::TC_BASES>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                             bnn::f4::Cfg<true, bnn::TC_BASES>::SMEM_BYTES) != cudaSuccess)
        return -1;
    cudaLaunchConfig_t cfg = {};
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeClusterDimension;
    attr[0].val.clusterDim.x = 2;
    attr[0].val.clusterDim.y = 1;
    attr[0].val.clusterDim.z = 1;
    cfg.gridDim = dim3(2 * 74);
    cfg.blockDim = dim3(C2::THREADS);
    cfg.dynamicSmemBytes = C2::SMEM_BYTES;
    cfg.attrs = attr;
    cfg.numAttrs = 1;
    int n = 0;
    if (cudaOccupancyMaxActiveClusters(&n, bnn::xnor_gemm_f4_kernel<true>, &cfg) != cudaSuccess) {
        cudaGetLastError();
        n = 0;
    }
    if (n < 1) n = kNoPairs;                                  // pairs unavailable: f4_plan never picks them
    if (dev < kMaxDevices) pairs[dev].store(n, std::memory_order_release);
    return n;
}

// Per-device one-time opt-in to the add table of the binary-weight GEMV.
bool bw_gemv_smem_configured() {
    constexpr int kMaxDevices = 64;
    static std::atomic<int> done[kMaxDevices];
    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess || dev < 0) return false;
    if (dev < kMaxDevices && done[dev].load(std::memory_order_acquire)) return true;
    const int bytes = bnn::bwg::smem_bytes(bnn::bwg::MAX_KW);
    if (cudaFuncSetAttribute(bnn::bw_gemv_kernel<float>, cudaFuncAttributeMaxDynamicSharedMemorySize, bytes) !=
            cudaSuccess ||
        cudaFuncSetAttribute(bnn::bw_gemv_kernel<__nv_bfloat16>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                             bytes) != cudaSuccess)
        return false;
    if (dev < kMaxDevices) done[dev].store(1, std::memory_order_release);
    return true;
}

// Opt the ternary GEMV (x staged in up to 96 KiB of shared memory) in once
// per device, for both block shapes the launcher uses.
bool ternary_gemv_smem_configured() {
    constexpr int kMaxDevices = 64;
    static std::atomic<int> done[kMaxDevices];
    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess || dev < 0) return false;
    if (dev < kMaxDevices && done[dev].load(std::memory_order_acquire)) return true;
    const int bytes = (int)(bnn::tgv::MAX_WORDS * 16);
    if (cudaFuncSetAttribute(bnn::ternary_gemv_i8_kernel<256, 4, 2>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                             bytes) != cudaSuccess ||
        cudaFuncSetAttribute(bnn::ternary_gemv_i8_kernel<256, 8, 2>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                             bytes) != cudaSuccess)
        return false;
    if (dev < kMaxDevices) done[dev].store(1, std::memory_order_release);
    return true;
}

std::atomic<int> g_gemm_engine{BNN_GEMM_ENGINE_AUTO};

int sm_count() {
    int dev = 0, sms = 148;
    if (cudaGetDevice(&dev) == cudaSuccess) cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);
    return sms;
}

bnn_status check_packed_operand(const uint32_t* p, int64_t ld, int64_t kw) {
    if (p == nullptr) return BNN_ERR_INVALID_ARG;
    if (ld < kw) return BNN_ERR_INVALID_ARG;
    if ((ld & 3) != 0 || !aligned(p, 16)) return BNN_ERR_ALIGNMENT;
    return BNN_OK;
}

bnn_status launch_gemm(const uint32_t* A, int64_t lda, const uint32_t* W, int64_t ldw, int64_t M, int64_t N,
                       int64_t K, const bnn::GemmEpilogue& ep, cudaStream_t stream) {
    using namespace bnn::gemm;
    const int64_t kw = packed_ld_words(K);
    CUtensorMap tmA, tmW;
    if (!encode_packed_map(&tmA, A, kw, M, lda, BM) || !encode_packed_map(&tmW, W, kw, N, ldw, BN))
        return BNN_ERR_CUDA;
    const int64_t tiles_n = ceil_div(N, BN);
    const int64_t tiles = ceil_div(M, BM) * tiles_n;
    if (tiles > INT_MAX) return BNN_ERR_INVALID_ARG;
    if (!gemm_smem_configured())
        return BNN_ERR_CUDA;
    bnn::GemmEpilogue e = ep;
    e.bits_words = packed_ld_words(N);
    bnn::xnor_gemm_popc_kernel<TN, CSA><<<(unsigned)tiles, THREADS, SMEM_BYTES, stream>>>(
        tmA, tmW, (int)M, (int)N, (int)K, (int)kw, (int)tiles_n, e);
    return launch_status();
}

bnn_status launch_gemm_tc(const uint32_t* A, int64_t lda, const uint32_t* W, int64_t ldw, int64_t M, int64_t N,
                          int64_t K, const bnn::GemmEpilogue& ep, cudaStream_t stream) {
    using namespace bnn::tc;
    const int64_t kw = packed_ld_words(K);
    CUtensorMap tmA, tmW;
    if (!encode_packed_map(&tmA, A, kw, M, lda, BM, BKW, CU_TENSOR_MAP_SWIZZLE_NONE) ||
        !encode_packed_map(&tmW, W, kw, N, ldw, BN, BKW, CU_TENSOR_MAP_SWIZZLE_NONE))
        return BNN_ERR_CUDA;
    const int64_t tiles_m = ceil_div(M, BM), tiles_n = ceil_div(N, BN);
    if (tiles_m * tiles_n > INT_MAX) return BNN_ERR_INVALID_ARG;
    if (!gemm_tc_smem_configured()) return BNN_ERR_CUDA;
    const int64_t grid = std::min<int64_t>(tiles_m * tiles_n, sm_count());
    bnn::GemmEpilogue e = ep;
    e.bits_words = packed_ld_words(N);
    bnn::xnor_gemm_tc_kernel<bnn::TC_BINARY><<<(unsigned)grid, THREADS, SMEM_BYTES, stream>>>(
        tmA, tmW, (int)M, (int)N, (int)K, (int)kw, (int)tiles_m, (int)tiles_n, e, bnn::TcPlanes{});
    return launch_status();
}

// 2-D map over a row-major fp32 / int32 output [rows, cols] with row stride
// ld elements, for 32 x 32 tensor stores from 128B-swizzled shared memory.
// False (store directly) when the pointer or the stride does not suit one.
bool encode_output_map(CUtensorMap* map, void* base, CUtensorMapDataType dt, int64_t cols, int64_t rows,
                       int64_t ld) {
    if (base == nullptr || !aligned(base, 16) || (ld * 4) % 16 != 0 || cols < 1 || rows < 1) return false;
    auto enc = tensor_map_encoder();
    if (enc == nullptr) return false;
    cuuint64_t dims[2] = {(cuuint64_t)cols, (cuuint64_t)rows};
    cuuint64_t strides[1] = {(cuuint64_t)ld * 4u};
    cuuint32_t box[2] = {32, 32};
    cuuint32_t estr[2] = {1, 1};
    return enc(map, dt, 2, base, dims, strides, box, estr, CU_TENSOR_MAP_INTERLEAVE_NONE,
               CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_NONE,
               CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

// Launch plan of the 4-bit kernel: single CTAs or CTA pairs, and the tile
// width bn (a multiple of 32 up to 224).  Shared-memory traffic bounds a
// stage: per SM it moves 128 + bn rows (single) or 128 + bn / 2 rows (pair)
// for the same 128 x bn x 256 multiply-adds, so the plan minimises (rounds
// of tiles over the resident CTAs or pairs) x (rows per stage).
struct F4Plan {
    bool pair;
    int bn;
};
F4Plan f4_plan(int64_t M, int64_t N, int64_t sms, int64_t pairs) {
    F4Plan best{false, bnn::f4::BN_MAX};
    int64_t best_cost = INT64_MAX;
    for (int pair = 0; pair < 2; ++pair) {
        if (pair && (pairs >= kNoPairs || M <= bnn::f4::BM)) continue;
        const int64_t units = pair ? pairs : sms;
        const int64_t tiles_m = ceil_div(M, (int64_t)bnn::f4::BM * (pair ? 2 : 1));
        for (int bn = bnn::f4::BN_MAX; bn >= 128; bn -= 32) {
            const int64_t tiles = tiles_m * ceil_div(N, bn);
            const int64_t cost = ceil_div(tiles, units) * (bnn::f4::BM + (pair ? bn / 2 : bn));
            if (cost < best_cost) {
                best_cost = cost;
                best = F4Plan{pair != 0, bn};
            }
        }
    }
    return best;
}

// Tile width of a CTA-pair e2m1 launch whose tiles hold bn / per_col output
// columns: the multiple of 32 up to 224 that minimises (rounds of tiles over
// the resident pairs) x (rows per stage, 128 + bn / 2).
int f4_pair_tile_n(int64_t tiles_m, int64_t N, int per_col, int64_t pairs) {
    int best = bnn::f4::BN_MAX;
    int64_t best_cost = INT64_MAX;
    for (int bn = bnn::f4::BN_MAX; bn >= 128; bn -= 32) {
        const int64_t tiles = tiles_m * ceil_div(N, (int64_t)(bn / per_col));
        const int64_t cost = ceil_div(tiles, pairs) * (bnn::f4::BM + bn / 2);
        if (cost < best_cost) {
            best_cost = cost;
            best = bn;
        }
    }
    return best;
}

// One launch of the CTA-pair e2m1 kernel: clusters of two, as many as are
// resident at once (the tiles are walked persistently).
template <int MODE>
bnn_status launch_f4_pairs(const CUtensorMap& tmA, const CUtensorMap& tmW, const CUtensorMap& tmCi,
                           const CUtensorMap& tmCf, int64_t M, int64_t N, int64_t K, int64_t kw, int bn, int64_t tiles_m,
                           int64_t tiles_n, int tma_out, const bnn::GemmEpilogue& e, const bnn::TcPlanes& pl,
                           int pairs, cudaStream_t stream) {
    using C = bnn::f4::Cfg<true, MODE>;
    const int64_t clusters = std::min<int64_t>(tiles_m * tiles_n, pairs);
    cudaLaunchConfig_t cfg = {};
    cudaLaunchAttribute attr[2];
    attr[0].id = cudaLaunchAttributeClusterDimension;
    attr[0].val.clusterDim.x = 2;
    attr[0].val.clusterDim.y = 1;
    attr[0].val.clusterDim.z = 1;
    // The kernel's set-up may overlap the previous kernel's last tiles; its
    // loads and stores wait for that kernel (griddepcontrol.wait).
    attr[1].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    attr[1].val.programmaticStreamSerializationAllowed = 1;
    cfg.gridDim = dim3((unsigned)(2 * clusters));
    cfg.blockDim = dim3(C::THREADS);
    cfg.dynamicSmemBytes = C::SMEM_BYTES;
    cfg.stream = stream;
    cfg.attrs = attr;
    cfg.numAttrs = 2;
    if (cudaLaunchKernelEx(&cfg, bnn::xnor_gemm_f4_kernel<true, MODE>, tmA, tmW, tmCi, tmCf, (int)M, (int)N, (int)K,
                           (int)kw, bn, (int)tiles_m, (int)tiles_n, tma_out, e, pl) != cudaSuccess)
        return BNN_ERR_CUDA;
    return launch_status();
}

// The +1/-1 product on the tensor cores with e2m1 operands.  Callers check
// K against MAX_KP (the exact-integer range of the fp32 accumulator).
bnn_status launch_gemm_f4(const uint32_t* A, int64_t lda, const uint32_t* W, int64_t ldw, int64_t M, int64_t N,
                          int64_t K, const bnn::GemmEpilogue& ep, cudaStream_t stream) {
    using namespace bnn::f4;
    const int64_t kw = packed_ld_words(K);
    const int64_t sms = sm_count();
    const int pairs = gemm_f4_pairs_resident();
    if (pairs < 0) return BNN_ERR_CUDA;
    const F4Plan plan = f4_plan(M, N, sms, pairs);
    const int bn = plan.bn, ctas = plan.pair ? 2 : 1;
    // Packed words per row per stage (two K atoms in CTA pairs) and the
    // matching TMA swizzle of the packed rows (32 or 64 bytes).
    const int sbkw = plan.pair ? Cfg<true>::S_BKW : Cfg<false>::S_BKW;
    const CUtensorMapSwizzle psw = sbkw == 16 ? CU_TENSOR_MAP_SWIZZLE_64B : CU_TENSOR_MAP_SWIZZLE_32B;
    CUtensorMap tmA, tmW;
    if (!encode_packed_map(&tmA, A, kw, M, lda, BM, sbkw, psw) ||
        !encode_packed_map(&tmW, W, kw, N, ldw, bn / ctas, sbkw, psw))
        return BNN_ERR_CUDA;
    const int64_t tiles_m = ceil_div(M, (int64_t)BM * ctas), tiles_n = ceil_div(N, bn);
    if (tiles_m * tiles_n > INT_MAX) return BNN_ERR_INVALID_ARG;
    bnn::GemmEpilogue e = ep;
    e.bits_words = packed_ld_words(N);
    // Dense outputs leave through TMA tensor stores where a map fits them.
    CUtensorMap tmCi, tmCf;
    std::memset(&tmCi, 0, sizeof(tmCi));
    std::memset(&tmCf, 0, sizeof(tmCf));
    int tma_out = 0;
    if (encode_output_map(&tmCi, e.c_i32, CU_TENSOR_MAP_DATA_TYPE_INT32, N, M, e.ldc)) tma_out |= 1;
    if (encode_output_map(&tmCf, e.c_f32, CU_TENSOR_MAP_DATA_TYPE_FLOAT32, N, M, e.ldf)) tma_out |= 2;
    if (!plan.pair) {
        const int64_t grid = std::min<int64_t>(tiles_m * tiles_n, sms);
        bnn::xnor_gemm_f4_kernel<false><<<(unsigned)grid, Cfg<false>::THREADS, Cfg<false>::SMEM_BYTES, stream>>>(
            tmA, tmW, tmCi, tmCf, (int)M, (int)N, (int)K, (int)kw, bn, (int)tiles_m, (int)tiles_n, tma_out, e,
            bnn::TcPlanes{});
        return launch_status();
    }
    return launch_f4_pairs<bnn::TC_BINARY>(tmA, tmW, tmCi, tmCf, M, N, K, kw, bn, tiles_m, tiles_n, tma_out, e,
                                           bnn::TcPlanes{}, pairs, stream);
}

// Padded K of the 4-bit kernel: K rounded up to whole stages, taken at the
// largest stage (two K atoms, 512 elements) so that the bound holds for
// every launch plan.
inline int64_t f4_padded_k(int64_t K) {
    return ceil_div(packed_ld_words(K), (int64_t)2 * bnn::f4::BKW) * 2 * bnn::f4::BKE;
}

// 3-D map over a plane-interleaved packed matrix (plane p of row r is packed
// row r * planes + p): dimensions (word, plane, row), box (4 words,
// box_planes, box_rows), no swizzle.  box_planes > planes reads the missing
// planes as zero words.
bool encode_plane_map(CUtensorMap* map, const uint32_t* base, int64_t kw, int64_t planes, int64_t rows, int64_t ld,
                      int box_planes, int box_rows, int box_words = bnn::tc::BKW,
                      CUtensorMapSwizzle swizzle = CU_TENSOR_MAP_SWIZZLE_NONE) {
    auto enc = tensor_map_encoder();
    if (enc == nullptr) return false;
    cuuint64_t dims[3] = {(cuuint64_t)kw, (cuuint64_t)planes, (cuuint64_t)rows};
    cuuint64_t strides[2] = {(cuuint64_t)ld * 4u, (cuuint64_t)(planes * ld) * 4u};
    cuuint32_t box[3] = {(cuuint32_t)box_words, (cuuint32_t)box_planes, (cuuint32_t)box_rows};
    cuuint32_t estr[3] = {1, 1, 1};
    CUresult r = enc(map, CU_TENSOR_MAP_DATA_TYPE_UINT32, 3, const_cast<uint32_t*>(base), dims, strides, box, estr,
                     CU_TENSOR_MAP_INTERLEAVE_NONE, swizzle, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
                     CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
    return r == CUDA_SUCCESS;
}

int pow2_at_least(int v) {
    int p = 1;
    while (p < v) p <<= 1;
    return p;
}

// Engine for one product: the tensor cores once the tile is reasonably
// filled (M >= 128, N >= 128, K >= 512); the integer pipes otherwise.  The
// tensor engine multiplies e2m1 operands while the padded K keeps every
// partial sum exact in fp32, and int8 operands beyond (or when forced).
bnn_status dispatch_gemm(const uint32_t* A, int64_t lda, const uint32_t* W, int64_t ldw, int64_t M, int64_t N,
                         int64_t K, const bnn::GemmEpilogue& ep, cudaStream_t stream) {
    int engine = g_gemm_engine.load(std::memory_order_relaxed);
    if (engine == BNN_GEMM_ENGINE_AUTO)
        engine = (M >= 128 && N >= 128 && K >= 512) ? BNN_GEMM_ENGINE_TENSOR : BNN_GEMM_ENGINE_POPCOUNT;
    if (engine == BNN_GEMM_ENGINE_TENSOR && f4_padded_k(K) <= bnn::f4::MAX_KP)
        return launch_gemm_f4(A, lda, W, ldw, M, N, K, ep, stream);
    if (engine == BNN_GEMM_ENGINE_TENSOR || engine == BNN_GEMM_ENGINE_TENSOR_I8)
        return launch_gemm_tc(A, lda, W, ldw, M, N, K, ep, stream);
    return launch_gemm(A, lda, W, ldw, M, N, K, ep, stream);
}

bnn_status check_gemm_dims(int64_t M, int64_t N, int64_t K) {
    if (M < 0 || N < 0 || K < 1) return BNN_ERR_INVALID_ARG;
    if (M > INT_MAX || N > INT_MAX || K > (INT_MAX / 2)) return BNN_ERR_INVALID_ARG;
    return BNN_OK;
}

template <typename XT>
bnn_status launch_gemv_t(const uint32_t* W, int64_t ldw, const XT* x, int64_t N, int64_t K, int64_t kw,
                         const float* alpha, int32_t* y_i32, float* y_f32, bool weights_static,
                         bool inputs_static, bool independent, cudaStream_t stream) {
    using namespace bnn::gemv;
    const int64_t nchunks = kw / 4;
    int lpr = 1;
    while (lpr < 32 && lpr < nchunks) lpr <<= 1;
    const int64_t rows_per_block = (int64_t)WARPS * U * (32 / lpr);
    const int64_t blocks = ceil_div(N, rows_per_block);
    const size_t smem = (size_t)kw * 4;

    cudaLaunchConfig_t cfg{};
    cfg.gridDim = dim3((unsigned)blocks);
    cfg.blockDim = dim3(THREADS);
    cfg.dynamicSmemBytes = smem;
    cfg.stream = stream;
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    attr[0].val.programmaticStreamSerializationAllowed = 1;
    cfg.attrs = attr;
    cfg.numAttrs = 1;

    cudaError_t e = cudaSuccess;
    const int iN = (int)N, iK = (int)K, ikw = (int)kw;
    const bool single = nchunks <= lpr;
    if ((int64_t)blocks * rows_per_block > (int64_t)INT_MAX) return BNN_ERR_INVALID_ARG;
    auto launch = [&](auto kern) -> bnn_status {
        if (smem > 48 * 1024 &&
            cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem) != cudaSuccess)
            return BNN_ERR_CUDA;
        e = cudaLaunchKernelEx(&cfg, kern, W, ldw, x, iN, iK, ikw, alpha, y_i32, y_f32, 1);
        return BNN_OK;
    };
    bnn_status st = BNN_OK;
    const bool vec = aligned(x, 16);
    if (lpr == 32 && single && vec) {
        // Rows of 68..128 words: the dedicated one-chunk-per-lane kernel.  Its
        // block shape depends on what the launch may overlap; each was the
        // fastest of ~30 shapes on the 11008 x 4096 decode GEMV in back-to-back
        // launches (steps of 1.10 / 1.39 / 2.18 us):
        //   all three flags (nothing to wait for):  256 threads x 12 rows per warp
        //   static W and x, ordered store:          128 threads x 8 rows per warp
        //   x (or W) read after the wait:           768 threads x 2 rows per warp
        auto go = [&](auto kern, int th, int u) -> bnn_status {
            const int64_t rows = (int64_t)(th / 32) * u;
            cfg.gridDim = dim3((unsigned)ceil_div(N, rows));
            cfg.blockDim = dim3((unsigned)th);
            e = cudaLaunchKernelEx(&cfg, kern, W, ldw, x, iN, iK, ikw, alpha, y_i32, y_f32, weights_static ? 1 : 0,
                                   inputs_static ? 1 : 0, independent ? 2 : 1);
            if (e != cudaSuccess) return BNN_ERR_CUDA;
            return launch_status();
        };
        if (independent) return go(bnn::xnor_gemv_row128_kernel<XT, 256, 12>, 256, 12);
        if (weights_static && inputs_static) return go(bnn::xnor_gemv_row128_kernel<XT, 128, 8>, 128, 8);
        return go(bnn::xnor_gemv_row128_kernel<XT, 768, 2>, 768, 2);
    }
#define BNN_GEMV_PICK(L, S, P)                                                                      \
    (vec ? launch(bnn::xnor_gemv_kernel<XT, L, S, P, true>) : launch(bnn::xnor_gemv_kernel<XT, L, S, P, false>))
#define BNN_GEMV_CASE(L)                                                                            \
    case L:                                                                                         \
        if (single)                                                                                 \
            st = weights_static ? BNN_GEMV_PICK(L, true, true) : BNN_GEMV_PICK(L, true, false);     \
        else                                                                                        \
            st = weights_static ? BNN_GEMV_PICK(L, false, true) : BNN_GEMV_PICK(L, false, false);   \
        break;
    switch (lpr) {
        BNN_GEMV_CASE(1)
        BNN_GEMV_CASE(2)
        BNN_GEMV_CASE(4)
        BNN_GEMV_CASE(8)
        BNN_GEMV_CASE(16)
        BNN_GEMV_CASE(32)
        default: return BNN_ERR_UNSUPPORTED;
    }
    if (st != BNN_OK) return st;
#undef BNN_GEMV_CASE
#undef BNN_GEMV_PICK
    if (e != cudaSuccess) return BNN_ERR_CUDA;
    return launch_status();
}

constexpr int64_t kGemvMaxWords = 48 * 1024;   // packed x in shared memory: <= 192 KiB

bnn_status gemv_impl(const uint32_t* W, int64_t ldw, const void* x, bnn_dtype x_dt, int64_t N, int64_t K,
                     const float* alpha, int32_t* y_i32, float* y_f32, bool weights_static,
                     bool inputs_static, bool independent, bnn_stream_t stream) {
    if (N < 0 || K < 1 || N > INT_MAX || K > INT_MAX / 2) return BNN_ERR_INVALID_ARG;
    if (x == nullptr || (y_i32 == nullptr && y_f32 == nullptr)) return BNN_ERR_INVALID_ARG;
    if (y_f32 != nullptr && alpha == nullptr) return BNN_ERR_INVALID_ARG;
    if (x_dt != BNN_F32 && x_dt != BNN_BF16) return BNN_ERR_INVALID_ARG;
    const int64_t kw = packed_ld_words(K);
    bnn_status st = check_packed_operand(W, ldw, kw);
    if (st != BNN_OK) return st;
    if (kw > kGemvMaxWords) return BNN_ERR_UNSUPPORTED;
    if (!aligned(x, x_dt == BNN_F32 ? 4 : 2)) return BNN_ERR_ALIGNMENT;
    if (N == 0) return BNN_OK;
    if (x_dt == BNN_F32)
        return launch_gemv_t(W, ldw, static_cast<const float*>(x), N, K, kw, alpha, y_i32, y_f32,
                             weights_static, inputs_static, independent, as_cuda(stream));
    return launch_gemv_t(W, ldw, static_cast<const __nv_bfloat16*>(x), N, K, kw, alpha, y_i32, y_f32,
                         weights_static, inputs_static, independent, as_cuda(stream));
}

// The device address of a host buffer that the device can access (pinned
// memory from cudaHostAlloc / cudaMallocHost or cudaHostRegister, mapped
// into the unified address space), else nullptr (pageable memory).
void* mapped_host_view(const void* p) {
    cudaPointerAttributes a{};
    if (cudaPointerGetAttributes(&a, p) != cudaSuccess) {
        cudaGetLastError();
        return nullptr;
    }
    return a.type == cudaMemoryTypeHost ? a.devicePointer : nullptr;
}

// copy16_kernel with programmatic dependent launch, enough blocks for one
// pass of VEC vectors per thread (capped).
template <bool SRC_EARLY>
bnn_status launch_copy16(const void* src, void* dst, size_t n16, cudaStream_t stream) {
    if (n16 == 0) return BNN_OK;
    const int64_t per_block = (int64_t)bnn::hostio::THREADS * bnn::hostio::VEC;
    const int64_t blocks = std::min<int64_t>(ceil_div((int64_t)n16, per_block), bnn::hostio::MAX_BLOCKS);
    cudaLaunchConfig_t cfg{};
    cfg.gridDim = dim3((unsigned)blocks);
    cfg.blockDim = dim3(bnn::hostio::THREADS);
    cfg.stream = stream;
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    attr[0].val.programmaticStreamSerializationAllowed = 1;
    cfg.attrs = attr;
    cfg.numAttrs = 1;
    if (cudaLaunchKernelEx(&cfg, bnn::copy16_kernel<SRC_EARLY>, static_cast<const uint4*>(src),
                           static_cast<uint4*>(dst), (int64_t)n16) != cudaSuccess)
        return BNN_ERR_CUDA;
    return BNN_OK;
}

}  // namespace

extern "C" {

bnn_status bnn_set_gemm_engine(int engine) {
    if (engine != BNN_GEMM_ENGINE_AUTO && engine != BNN_GEMM_ENGINE_POPCOUNT && engine != BNN_GEMM_ENGINE_TENSOR &&
        engine != BNN_GEMM_ENGINE_TENSOR_I8)
        return BNN_ERR_INVALID_ARG;
    g_gemm_engine.store(engine, std::memory_order_relaxed);
    return BNN_OK;
}

int bnn_get_gemm_engine(void) { return g_gemm_engine.load(std::memory_order_relaxed); }

int64_t bnn_packed_ld_words(int64_t K) { return K < 1 ? -1 : packed_ld_words(K); }

int64_t bnn_conv3x3_ld_words(int64_t cin) {
    if (cin < 1) return -1;
    return (9 * ((cin + 31) / 32) + 3) / 4 * 4;
}

const char* bnn_status_string(int status) {
    switch (status) {
        case BNN_OK: return "ok";
        case BNN_ERR_INVALID_ARG: return "invalid argument";
        case BNN_ERR_ALIGNMENT: return "pointer or leading dimension not aligned";
        case BNN_ERR_UNSUPPORTED: return "unsupported shape, dtype or mode";
        case BNN_ERR_CUDA: return "CUDA error";
        case BNN_ERR_DEVICE_TIMEOUT: return "a kernel gave up waiting on an asynchronous copy";
        default: return "unknown status";
    }
}

bnn_status bnn_device_error(int32_t* code_out) {
    if (code_out == nullptr) return BNN_ERR_INVALID_ARG;
    if (cudaDeviceSynchronize() != cudaSuccess) return BNN_ERR_CUDA;
    int v = 0;
    if (cudaMemcpyFromSymbol(&v, bnn::g_device_error, sizeof(int)) != cudaSuccess) return BNN_ERR_CUDA;
    if (v != 0) {
        const int zero = 0;
        if (cudaMemcpyToSymbol(bnn::g_device_error, &zero, sizeof(int)) != cudaSuccess) return BNN_ERR_CUDA;
    }
    *code_out = v;
    return BNN_OK;
}

bnn_status bnn_probe_int_pipes(int64_t iters, double* popc_per_clk_sm, double* lop3_per_clk_sm,
                               double* csa_words_per_clk_sm) {
    if (iters < 1 || iters > (1 << 24) || popc_per_clk_sm == nullptr || lop3_per_clk_sm == nullptr ||
        csa_words_per_clk_sm == nullptr)
        return BNN_ERR_INVALID_ARG;
    const int sms = sm_count();
    if (sms < 1 || sms > bnn::probe::MAX_SMS) return BNN_ERR_UNSUPPORTED;
    void (*kern[bnn::probe::MODES])(int, uint32_t) = {bnn::int_pipe_probe_kernel<0>, bnn::int_pipe_probe_kernel<1>,
                                                      bnn::int_pipe_probe_kernel<2>};
    // Operations each thread retires per loop iteration: 4 x 8 POPC, 4 x 8
    // LOP3, and 4 accumulators x 8 words.
    const double per_iter[bnn::probe::MODES] = {32.0, 32.0, 32.0};
    double* out[bnn::probe::MODES] = {popc_per_clk_sm, lop3_per_clk_sm, csa_words_per_clk_sm};
    unsigned long long cyc[bnn::probe::MAX_SMS];
    for (int m = 0; m < bnn::probe::MODES; ++m) {
        if (cudaFuncSetAttribute(kern[m], cudaFuncAttributeMaxDynamicSharedMemorySize, bnn::probe::SMEM_BYTES) !=
            cudaSuccess)
            return BNN_ERR_CUDA;
        kern[m]<<<sms, bnn::probe::THREADS, bnn::probe::SMEM_BYTES>>>((int)iters, 0x2545F491u);
        if (cudaGetLastError() != cudaSuccess || cudaDeviceSynchronize() != cudaSuccess) return BNN_ERR_CUDA;
        if (cudaMemcpyFromSymbol(cyc, bnn::g_probe_cycles, sizeof(unsigned long long) * (size_t)sms) != cudaSuccess)
            return BNN_ERR_CUDA;
        std::sort(cyc, cyc + sms);
        const double median = (double)cyc[sms / 2];
        if (median <= 0.0) return BNN_ERR_CUDA;
        *out[m] = (double)bnn::probe::THREADS * (double)iters * per_iter[m] / median;
    }
    return BNN_OK;
}

bnn_status bnn_selftest_wait_timeout(int64_t timeout_ns, int32_t* waited_out) {
    if (timeout_ns < 1 || timeout_ns > 10000000000LL || waited_out == nullptr) return BNN_ERR_INVALID_ARG;
    bnn::wait_timeout_selftest_kernel<<<1, 32>>>((unsigned long long)timeout_ns);
    int h = -1;
    if (cudaGetLastError() != cudaSuccess || cudaDeviceSynchronize() != cudaSuccess ||
        cudaMemcpyFromSymbol(&h, bnn::g_selftest_result, sizeof(int)) != cudaSuccess)
        return BNN_ERR_CUDA;
    *waited_out = (h == 0) ? 1 : 0;
    return BNN_OK;
}

namespace {

bnn_status pack_sign_rows(const void* x, bnn_dtype dt, int64_t rows, int64_t K, int64_t ld_x, const float* beta,
                          uint32_t* packed, int64_t ld_words, float* alpha_out, bnn_stream_t stream) {
    if (x == nullptr || packed == nullptr) return BNN_ERR_INVALID_ARG;
    if (rows < 0 || K < 1 || ld_x < K) return BNN_ERR_INVALID_ARG;
    if (dt != BNN_F32 && dt != BNN_BF16) return BNN_ERR_INVALID_ARG;
    const int64_t kw = packed_ld_words(K);
    if (ld_words < kw) return BNN_ERR_INVALID_ARG;
    if ((ld_words & 3) != 0 || !aligned(packed, 16)) return BNN_ERR_ALIGNMENT;
    const size_t es = dt == BNN_F32 ? 4 : 2;
    if (!aligned(x, es) || (alpha_out != nullptr && !aligned(alpha_out, 4))) return BNN_ERR_ALIGNMENT;
    if (beta != nullptr && !aligned(beta, 4)) return BNN_ERR_ALIGNMENT;
    if (rows == 0) return BNN_OK;
    const bool vec_ok = aligned(x, 16) && ((ld_x * (int64_t)es) % 16 == 0);
    const int64_t blocks = ceil_div(rows, 8);
    if (blocks > INT_MAX) return BNN_ERR_INVALID_ARG;
    cudaStream_t s = as_cuda(stream);
    const float* xf = static_cast<const float*>(x);
    const __nv_bfloat16* xb = static_cast<const __nv_bfloat16*>(x);
    const unsigned g = (unsigned)blocks;
    if (dt == BNN_F32 && beta == nullptr)
        bnn::pack_sign_rows_kernel<float, 4, false><<<g, 256, 0, s>>>(xf, rows, K, ld_x, packed, ld_words, alpha_out,
                                                                      kw, vec_ok, beta);
    else if (dt == BNN_F32)
        bnn::pack_sign_rows_kernel<float, 4, true><<<g, 256, 0, s>>>(xf, rows, K, ld_x, packed, ld_words, alpha_out,
                                                                     kw, vec_ok, beta);
    else if (beta == nullptr)
        bnn::pack_sign_rows_kernel<__nv_bfloat16, 4, false><<<g, 256, 0, s>>>(xb, rows, K, ld_x, packed, ld_words,
                                                                              alpha_out, kw, vec_ok, beta);
    else
        bnn::pack_sign_rows_kernel<__nv_bfloat16, 4, true><<<g, 256, 0, s>>>(xb, rows, K, ld_x, packed, ld_words,
                                                                             alpha_out, kw, vec_ok, beta);
    return launch_status();
}

// The TMA-streamed NCHW pack (pack_sign_nchw_tma_kernel): a 2-D map over
// the tensor as [n*c rows, hw pixels], box 32 rows x 128 bytes, zero fill
// past either end.  Returns UNSUPPORTED when the map cannot be encoded, so
// the caller falls back to the register kernel.
bnn_status pack_sign_nchw_tma(const void* x, bnn_dtype dt, int64_t n, int64_t c, int64_t hw, int64_t cw,
                              const float* beta, uint32_t* packed_nhwc, cudaStream_t s) {
    using namespace bnn::nchw_tma;
    auto enc = tensor_map_encoder();
    if (enc == nullptr) return BNN_ERR_UNSUPPORTED;
    const int64_t es = dt == BNN_F32 ? 4 : 2;
    const int64_t P = 128 / es;
    CUtensorMap map;
    cuuint64_t dims[2] = {(cuuint64_t)hw, (cuuint64_t)(n * c)};
    cuuint64_t strides[1] = {(cuuint64_t)(hw * es)};
    cuuint32_t box[2] = {(cuuint32_t)P, 32u};
    cuuint32_t estr[2] = {1, 1};
    if (enc(&map, dt == BNN_F32 ? CU_TENSOR_MAP_DATA_TYPE_UINT32 : CU_TENSOR_MAP_DATA_TYPE_UINT16, 2,
            const_cast<void*>(x), dims, strides, box, estr, CU_TENSOR_MAP_INTERLEAVE_NONE,
            CU_TENSOR_MAP_SWIZZLE_NONE, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
            CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) != CUDA_SUCCESS)
        return BNN_ERR_UNSUPPORTED;
    const int64_t tiles_per_plane = ceil_div(hw, P);
    const int64_t total = n * cw * tiles_per_plane;
    const int64_t blocks = std::min<int64_t>(sm_count(), ceil_div(total, WARPS));
    // one-time opt-in to the shared memory per device (kept out of captured graphs)
    {
        constexpr int kMaxDevices = 64;
        static std::atomic<int> done[kMaxDevices];
        int dev = 0;
        if (cudaGetDevice(&dev) != cudaSuccess || dev < 0) return BNN_ERR_CUDA;
        if (dev >= kMaxDevices || !done[dev].load(std::memory_order_acquire)) {
            if (cudaFuncSetAttribute(bnn::pack_sign_nchw_tma_kernel<float, false>,
                                     cudaFuncAttributeMaxDynamicSharedMemorySize, SMEM_BYTES) != cudaSuccess ||
                cudaFuncSetAttribute(bnn::pack_sign_nchw_tma_kernel<float, true>,
                                     cudaFuncAttributeMaxDynamicSharedMemorySize, SMEM_BYTES) != cudaSuccess ||
                cudaFuncSetAttribute(bnn::pack_sign_nchw_tma_kernel<__nv_bfloat16, false>,
                                     cudaFuncAttributeMaxDynamicSharedMemorySize, SMEM_BYTES) != cudaSuccess ||
                cudaFuncSetAttribute(bnn::pack_sign_nchw_tma_kernel<__nv_bfloat16, true>,
                                     cudaFuncAttributeMaxDynamicSharedMemorySize, SMEM_BYTES) != cudaSuccess)
                return BNN_ERR_CUDA;
            if (dev < kMaxDevices) done[dev].store(1, std::memory_order_release);
        }
    }
    auto go = [&](auto kern) -> bnn_status {
        kern<<<(unsigned)blocks, THREADS, SMEM_BYTES, s>>>(map, n, c, hw, cw, tiles_per_plane, packed_nhwc, beta);
        return launch_status();
    };
    if (dt == BNN_F32)
        return beta == nullptr ? go(bnn::pack_sign_nchw_tma_kernel<float, false>)
                               : go(bnn::pack_sign_nchw_tma_kernel<float, true>);
    return beta == nullptr ? go(bnn::pack_sign_nchw_tma_kernel<__nv_bfloat16, false>)
                           : go(bnn::pack_sign_nchw_tma_kernel<__nv_bfloat16, true>);
}

bnn_status pack_sign_nchw(const void* x, bnn_dtype dt, int64_t n, int64_t c, int64_t h, int64_t w, const float* beta,
                          uint32_t* packed_nhwc, bnn_stream_t stream) {
    if (x == nullptr || packed_nhwc == nullptr) return BNN_ERR_INVALID_ARG;
    if (n < 0 || c < 1 || h < 1 || w < 1) return BNN_ERR_INVALID_ARG;
    if (dt != BNN_F32 && dt != BNN_BF16) return BNN_ERR_INVALID_ARG;
    const size_t es = dt == BNN_F32 ? 4 : 2;
    if (!aligned(x, es) || !aligned(packed_nhwc, 4)) return BNN_ERR_ALIGNMENT;
    if (beta != nullptr && !aligned(beta, 4)) return BNN_ERR_ALIGNMENT;
    if (n == 0) return BNN_OK;
    const int64_t hw = h * w, cw = (c + 31) / 32;
    cudaStream_t s = as_cuda(stream);
    // TMA-streamed kernel: needs a 16-byte aligned tensor whose channel rows
    // are whole 16-byte units (TMA's stride rule) and coordinates in int32.
    if (aligned(x, 16) && (hw * (int64_t)es) % 16 == 0 && n * c < (int64_t)INT_MAX && hw < (int64_t)INT_MAX) {
        const bnn_status st = pack_sign_nchw_tma(x, dt, n, c, hw, cw, beta, packed_nhwc, s);
        if (st != BNN_ERR_UNSUPPORTED) return st;
    }
    const int64_t warps = n * ceil_div(hw, 8 * (int64_t)(16 / es)) * cw;   // (image, 8 vectors of pixels, word)
    const int64_t blocks = ceil_div(warps, 8);
    if (blocks > INT_MAX) return BNN_ERR_INVALID_ARG;
    const bool vec_ok = aligned(x, 16) && (hw % (int64_t)(16 / es) == 0);
    const float* xf = static_cast<const float*>(x);
    const __nv_bfloat16* xb = static_cast<const __nv_bfloat16*>(x);
    const unsigned g = (unsigned)blocks;
    if (dt == BNN_F32 && beta == nullptr)
        bnn::pack_sign_nchw_kernel<float, false><<<g, 256, 0, s>>>(xf, n, c, hw, cw, packed_nhwc, vec_ok, beta);
    else if (dt == BNN_F32)
        bnn::pack_sign_nchw_kernel<float, true><<<g, 256, 0, s>>>(xf, n, c, hw, cw, packed_nhwc, vec_ok, beta);
    else if (beta == nullptr)
        bnn::pack_sign_nchw_kernel<__nv_bfloat16, false><<<g, 256, 0, s>>>(xb, n, c, hw, cw, packed_nhwc, vec_ok, beta);
    else
        bnn::pack_sign_nchw_kernel<__nv_bfloat16, true><<<g, 256, 0, s>>>(xb, n, c, hw, cw, packed_nhwc, vec_ok, beta);
    return launch_status();
}

}  // namespace

bnn_status bnn_pack_sign(const void* x, bnn_dtype dt, int64_t rows, int64_t K, int64_t ld_x, uint32_t* packed,
                         int64_t ld_words, float* alpha_out, bnn_stream_t stream) {
    return pack_sign_rows(x, dt, rows, K, ld_x, nullptr, packed, ld_words, alpha_out, stream);
}

bnn_status bnn_pack_sign_rsign(const void* x, bnn_dtype dt, int64_t rows, int64_t K, int64_t ld_x, const float* beta,
                               uint32_t* packed, int64_t ld_words, bnn_stream_t stream) {
    if (beta == nullptr) return BNN_ERR_INVALID_ARG;
    return pack_sign_rows(x, dt, rows, K, ld_x, beta, packed, ld_words, nullptr, stream);
}

bnn_status bnn_pack_sign_nchw_rsign(const void* x, bnn_dtype dt, int64_t n, int64_t c, int64_t h, int64_t w,
                                    const float* beta, uint32_t* packed_nhwc, bnn_stream_t stream) {
    if (beta == nullptr) return BNN_ERR_INVALID_ARG;
    return pack_sign_nchw(x, dt, n, c, h, w, beta, packed_nhwc, stream);
}

bnn_status bnn_pack_sign_nchw(const void* x, bnn_dtype dt, int64_t n, int64_t c, int64_t h, int64_t w,
                              uint32_t* packed_nhwc, bnn_stream_t stream) {
    return pack_sign_nchw(x, dt, n, c, h, w, nullptr, packed_nhwc, stream);
}

bnn_status bnn_pack_conv3x3_weights(const void* w_oihw, bnn_dtype dt, int64_t cout, int64_t cin,
                                    uint32_t* packed, int64_t ld_words, float* alpha_out, bnn_stream_t stream) {
    if (w_oihw == nullptr || packed == nullptr) return BNN_ERR_INVALID_ARG;
    if (cout < 0 || cin < 1) return BNN_ERR_INVALID_ARG;
    if (dt != BNN_F32 && dt != BNN_BF16) return BNN_ERR_INVALID_ARG;
    if (ld_words < bnn_conv3x3_ld_words(cin)) return BNN_ERR_INVALID_ARG;
    if ((ld_words & 3) != 0 || !aligned(packed, 16)) return BNN_ERR_ALIGNMENT;
    if (!aligned(w_oihw, dt == BNN_F32 ? 4 : 2)) return BNN_ERR_ALIGNMENT;
    if (cout == 0) return BNN_OK;
    const int64_t blocks = ceil_div(cout, 8);
    if (blocks > INT_MAX) return BNN_ERR_INVALID_ARG;
    cudaStream_t s = as_cuda(stream);
    if (dt == BNN_F32)
        bnn::pack_conv3x3_weights_kernel<float><<<(unsigned)blocks, 256, 0, s>>>(
            static_cast<const float*>(w_oihw), cout, cin, packed, ld_words, alpha_out);
    else
        bnn::pack_conv3x3_weights_kernel<__nv_bfloat16><<<(unsigned)blocks, 256, 0, s>>>(
            static_cast<const __nv_bfloat16*>(w_oihw), cout, cin, packed, ld_words, alpha_out);
    return launch_status();
}

bnn_status bnn_xnor_gemm(const uint32_t* A, int64_t lda, const uint32_t* W, int64_t ldw, int64_t M, int64_t N,
                         int64_t K, const float* alpha, int32_t* C_i32, int64_t ldc, float* C_f32, int64_t ldf,
                         bnn_stream_t stream) {
    bnn_status st = check_gemm_dims(M, N, K);
    if (st != BNN_OK) return st;
    const int64_t kw = packed_ld_words(K);
    if ((st = check_packed_operand(A, lda, kw)) != BNN_OK) return st;
    if ((st = check_packed_operand(W, ldw, kw)) != BNN_OK) return st;
    if (C_i32 == nullptr && C_f32 == nullptr) return BNN_ERR_INVALID_ARG;
    if (C_i32 != nullptr && ldc < N) return BNN_ERR_INVALID_ARG;
    if (C_f32 != nullptr && (ldf < N || alpha == nullptr)) return BNN_ERR_INVALID_ARG;
    if ((C_i32 && !aligned(C_i32, 4)) || (C_f32 && !aligned(C_f32, 4))) return BNN_ERR_ALIGNMENT;
    if (M == 0 || N == 0) return BNN_OK;
    bnn::GemmEpilogue ep{};
    ep.c_i32 = C_i32;
    ep.ldc = ldc;
    ep.c_f32 = C_f32;
    ep.ldf = ldf;
    ep.alpha = alpha;
    return dispatch_gemm(A, lda, W, ldw, M, N, K, ep, as_cuda(stream));
}

bnn_status bnn_xnor_gemv(const uint32_t* W, int64_t ldw, const void* x, bnn_dtype x_dt, int64_t N, int64_t K,
                         const float* alpha, int32_t* y_i32, float* y_f32, bnn_stream_t stream) {
    return gemv_impl(W, ldw, x, x_dt, N, K, alpha, y_i32, y_f32, false, false, false, stream);
}

bnn_status bnn_xnor_gemv_ex(const uint32_t* W, int64_t ldw, const void* x, bnn_dtype x_dt, int64_t N, int64_t K,
                            const float* alpha, int32_t* y_i32, float* y_f32, uint32_t flags,
                            bnn_stream_t stream) {
    constexpr uint32_t kAll = BNN_GEMV_WEIGHTS_STATIC | BNN_GEMV_INPUTS_STATIC | BNN_GEMV_OUTPUT_FREE;
    if ((flags & ~kAll) != 0) return BNN_ERR_INVALID_ARG;
    return gemv_impl(W, ldw, x, x_dt, N, K, alpha, y_i32, y_f32, (flags & BNN_GEMV_WEIGHTS_STATIC) != 0,
                     (flags & BNN_GEMV_INPUTS_STATIC) != 0, flags == kAll, stream);
}

bnn_status bnn_xnor_gemv_host(const uint32_t* W, int64_t ldw, const void* x_host, bnn_dtype x_dt, int64_t N,
                              int64_t K, const float* alpha, void* x_dev, float* y_dev, float* y_host, uint32_t flags,
                              bnn_stream_t stream) {
    if ((flags & ~(uint32_t)(BNN_GEMV_WEIGHTS_STATIC | BNN_GEMV_INPUTS_STATIC)) != 0) return BNN_ERR_INVALID_ARG;
    if (x_host == nullptr || x_dev == nullptr || y_dev == nullptr || y_host == nullptr || alpha == nullptr)
        return BNN_ERR_INVALID_ARG;
    if (N < 0 || K < 1 || N > INT_MAX / 2 || K > INT_MAX / 2) return BNN_ERR_INVALID_ARG;
    if (x_dt != BNN_F32 && x_dt != BNN_BF16) return BNN_ERR_INVALID_ARG;
    if (!aligned(x_dev, 16) || !aligned(y_dev, 4)) return BNN_ERR_ALIGNMENT;
    const size_t xbytes = (size_t)K * (x_dt == BNN_F32 ? 4 : 2), ybytes = (size_t)N * 4;
    cudaStream_t s = as_cuda(stream);
    // x_dev is written just before the GEMV: only the weights may be static.
    const uint32_t gemv_flags = flags & BNN_GEMV_WEIGHTS_STATIC;
    // Pinned host buffers that the device can address take the two copies as
    // small kernels chained to the GEMV (hostio.cuh); other host memory, and
    // sizes or alignments that 16-byte vectors do not fit, take the copy
    // engines.
    const void* x_map = mapped_host_view(x_host);
    void* y_map = mapped_host_view(y_host);
    if (x_map != nullptr && y_map != nullptr && aligned(x_map, 16) && aligned(y_map, 16) && aligned(y_dev, 16) &&
        xbytes % 16 == 0 && ybytes % 16 == 0) {
        // BNN_GEMV_INPUTS_STATIC: nothing in flight writes x_host, so the
        // copy-in may read it before the previous work on the stream ends.
        bnn_status st = (flags & BNN_GEMV_INPUTS_STATIC) ? launch_copy16<true>(x_map, x_dev, xbytes / 16, s)
                                                          : launch_copy16<false>(x_map, x_dev, xbytes / 16, s);
        if (st != BNN_OK) return st;
        if ((st = bnn_xnor_gemv_ex(W, ldw, x_dev, x_dt, N, K, alpha, nullptr, y_dev, gemv_flags, stream)) != BNN_OK)
            return st;
        return N > 0 ? launch_copy16<false>(y_dev, y_map, ybytes / 16, s) : BNN_OK;
    }
    if (cudaMemcpyAsync(x_dev, x_host, xbytes, cudaMemcpyHostToDevice, s) != cudaSuccess) return BNN_ERR_CUDA;
    const bnn_status st = bnn_xnor_gemv_ex(W, ldw, x_dev, x_dt, N, K, alpha, nullptr, y_dev, gemv_flags, stream);
    if (st != BNN_OK) return st;
    if (N > 0 && cudaMemcpyAsync(y_host, y_dev, ybytes, cudaMemcpyDeviceToHost, s) != cudaSuccess)
        return BNN_ERR_CUDA;
    return BNN_OK;
}

bnn_status bnn_binary_weight_gemv(const uint32_t* W, int64_t ldw, const void* x, bnn_dtype x_dt, int64_t N,
                                  int64_t K, const float* alpha, float* y, uint32_t flags, bnn_stream_t stream) {
    constexpr uint32_t kAll = BNN_GEMV_WEIGHTS_STATIC | BNN_GEMV_INPUTS_STATIC | BNN_GEMV_OUTPUT_FREE;
    if ((flags & ~kAll) != 0) return BNN_ERR_INVALID_ARG;
    if (x == nullptr || alpha == nullptr || y == nullptr) return BNN_ERR_INVALID_ARG;
    if (N < 0 || K < 1 || N > INT_MAX / 2 || K > INT_MAX / 2) return BNN_ERR_INVALID_ARG;
    if (x_dt != BNN_F32 && x_dt != BNN_BF16) return BNN_ERR_INVALID_ARG;
    const int64_t kw = packed_ld_words(K);
    bnn_status st = check_packed_operand(W, ldw, kw);
    if (st != BNN_OK) return st;
    if (kw > bnn::bwg::MAX_KW) return BNN_ERR_UNSUPPORTED;
    if (!aligned(x, x_dt == BNN_F32 ? 4 : 2) || !aligned(alpha, 4) || !aligned(y, 4)) return BNN_ERR_ALIGNMENT;
    if (N == 0) return BNN_OK;
    if (!bw_gemv_smem_configured()) return BNN_ERR_CUDA;
    // One batch of U row groups per warp covers N with this many CTAs; more
    // rows loop.  Two CTAs fit on an SM, so the grid is capped at two per SM.
    int64_t lpr = 1;
    while (lpr < 32 && lpr < kw / 4) lpr <<= 1;
    const int64_t rows_per_cta = (int64_t)bnn::bwg::WARPS * bnn::bwg::U * (32 / lpr);
    const int64_t blocks = std::min<int64_t>(ceil_div(N, rows_per_cta), 2 * (int64_t)sm_count());
    cudaLaunchConfig_t cfg{};
    cfg.gridDim = dim3((unsigned)blocks);
    cfg.blockDim = dim3(bnn::bwg::THREADS);
    cfg.dynamicSmemBytes = (size_t)bnn::bwg::smem_bytes((int)kw);
    cfg.stream = as_cuda(stream);
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    attr[0].val.programmaticStreamSerializationAllowed = 1;
    cfg.attrs = attr;
    cfg.numAttrs = 1;
    const int prefetch = (flags & BNN_GEMV_WEIGHTS_STATIC) ? 1 : 0;
    const int xstatic = (flags & BNN_GEMV_INPUTS_STATIC) ? 1 : 0;
    const int dependent = flags == kAll ? 2 : 1;
    cudaError_t e;
    if (x_dt == BNN_F32)
        e = cudaLaunchKernelEx(&cfg, bnn::bw_gemv_kernel<float>, W, ldw, static_cast<const float*>(x), (int)N, (int)K,
                               (int)kw, alpha, y, prefetch, xstatic, dependent);
    else
        e = cudaLaunchKernelEx(&cfg, bnn::bw_gemv_kernel<__nv_bfloat16>, W, ldw,
                               static_cast<const __nv_bfloat16*>(x), (int)N, (int)K, (int)kw, alpha, y, prefetch,
                               xstatic, dependent);
    if (e != cudaSuccess) return BNN_ERR_CUDA;
    return launch_status();
}

bnn_status bnn_pack_bit_planes(const uint8_t* codes, int64_t rows, int64_t K, int64_t ld_codes, int bits,
                               uint32_t* planes, int64_t ld_words, bnn_stream_t stream) {
    if (codes == nullptr || planes == nullptr) return BNN_ERR_INVALID_ARG;
    if (rows < 0 || K < 1 || ld_codes < K || bits < 1 || bits > 8) return BNN_ERR_INVALID_ARG;
    const int64_t kw = packed_ld_words(K);
    if (ld_words < kw) return BNN_ERR_INVALID_ARG;
    if ((ld_words & 3) != 0 || !aligned(planes, 16)) return BNN_ERR_ALIGNMENT;
    if (rows == 0) return BNN_OK;
    const int64_t blocks = ceil_div(rows, 8);
    if (blocks > INT_MAX) return BNN_ERR_INVALID_ARG;
    const bool vec = aligned(codes, 16) && (ld_codes % 16 == 0);
    bnn::pack_bit_planes_kernel<<<(unsigned)blocks, 256, 0, as_cuda(stream)>>>(codes, rows, K, ld_codes, bits, planes,
                                                                                ld_words, kw, vec);
    return launch_status();
}

bnn_status bnn_bitserial_gemm(const uint32_t* A, int64_t lda, int a_bits, const uint32_t* W, int64_t ldw, int w_bits,
                              int64_t M, int64_t N, int64_t K, const float* alpha, int32_t* C_i32, int64_t ldc,
                              float* C_f32, int64_t ldf, bnn_stream_t stream) {
    using namespace bnn::tc;
    bnn_status st = check_gemm_dims(M, N, K);
    if (st != BNN_OK) return st;
    if (a_bits < 1 || a_bits > MAX_CODE_PLANES || w_bits < 1 || w_bits > MAX_CODE_PLANES) return BNN_ERR_INVALID_ARG;
    // The int32 accumulator holds K * (2^a - 1) * (2^w - 1) at most.
    if ((double)K * (double)((1 << a_bits) - 1) * (double)((1 << w_bits) - 1) > (double)INT_MAX)
        return BNN_ERR_INVALID_ARG;
    if (M * a_bits > INT_MAX || N * w_bits > INT_MAX) return BNN_ERR_INVALID_ARG;
    const int64_t kw = packed_ld_words(K);
    if ((st = check_packed_operand(A, lda, kw)) != BNN_OK) return st;
    if ((st = check_packed_operand(W, ldw, kw)) != BNN_OK) return st;
    if (C_i32 == nullptr && C_f32 == nullptr) return BNN_ERR_INVALID_ARG;
    if (C_i32 != nullptr && ldc < N) return BNN_ERR_INVALID_ARG;
    if (C_f32 != nullptr && (ldf < N || alpha == nullptr)) return BNN_ERR_INVALID_ARG;
    if ((C_i32 && !aligned(C_i32, 4)) || (C_f32 && !aligned(C_f32, 4)) || (alpha && !aligned(alpha, 4)))
        return BNN_ERR_ALIGNMENT;
    if (M == 0 || N == 0) return BNN_OK;
    {
        // Codes of up to two bits are exact e2m1 values (code c as the value
        // c / 2): the e2m1 kernel in CTA pairs, while every partial sum times
        // 4 (at most 9 per element of the padded K) stays an integer the
        // epilogue converts exactly.
        const int engine = g_gemm_engine.load(std::memory_order_relaxed);
        const int pairs = engine == BNN_GEMM_ENGINE_TENSOR_I8 ? -1 : gemm_f4_pairs_resident();
        if (a_bits <= bnn::f4::MAX_F4_PLANES && w_bits <= bnn::f4::MAX_F4_PLANES && pairs > 0 && pairs < kNoPairs &&
            M > bnn::f4::BM && 9 * f4_padded_k(K) < (int64_t(1) << 22)) {
            const int bn = f4_pair_tile_n(ceil_div(M, (int64_t)2 * bnn::f4::BM), N, 1, pairs);
            CUtensorMap fA, fW, fCi, fCf;
            std::memset(&fCi, 0, sizeof(fCi));
            std::memset(&fCf, 0, sizeof(fCf));
            static_assert(bnn::f4::Cfg<true, bnn::TC_PLANE_CODES>::S_BKW == bnn::f4::BKW, "codes stage one K atom");
            if (!encode_plane_map(&fA, A, kw, a_bits, M, lda, a_bits, bnn::f4::BM, bnn::f4::BKW,
                                  CU_TENSOR_MAP_SWIZZLE_32B) ||
                !encode_plane_map(&fW, W, kw, w_bits, N, ldw, w_bits, bn / 2, bnn::f4::BKW, CU_TENSOR_MAP_SWIZZLE_32B))
                return BNN_ERR_CUDA;
            bnn::GemmEpilogue e{};
            e.c_i32 = C_i32;
            e.ldc = ldc;
            e.c_f32 = C_f32;
            e.ldf = ldf;
            e.alpha = alpha;
            e.bits_words = packed_ld_words(N);
            int tma_out = 0;
            if (encode_output_map(&fCi, C_i32, CU_TENSOR_MAP_DATA_TYPE_INT32, N, M, ldc)) tma_out |= 1;
            if (encode_output_map(&fCf, C_f32, CU_TENSOR_MAP_DATA_TYPE_FLOAT32, N, M, ldf)) tma_out |= 2;
            bnn::TcPlanes pl{};
            pl.ja = a_bits;
            pl.jw = w_bits;
            return launch_f4_pairs<bnn::TC_PLANE_CODES>(fA, fW, fCi, fCf, M, N, K, kw, bn,
                                                        ceil_div(M, (int64_t)2 * bnn::f4::BM), ceil_div(N, bn),
                                                        tma_out, e, pl, pairs, as_cuda(stream));
        }
    }
    CUtensorMap tmA, tmW;
    if (!encode_plane_map(&tmA, A, kw, a_bits, M, lda, a_bits, BM) ||
        !encode_plane_map(&tmW, W, kw, w_bits, N, ldw, w_bits, BN))
        return BNN_ERR_CUDA;
    const int64_t tiles_m = ceil_div(M, BM), tiles_n = ceil_div(N, BN);
    if (tiles_m * tiles_n > INT_MAX) return BNN_ERR_INVALID_ARG;
    if (!gemm_tc_smem_configured()) return BNN_ERR_CUDA;
    bnn::TcPlanes pl{};
    pl.ja = a_bits;
    pl.jw = w_bits;
    pl.j_real = a_bits;
    pl.i_real = w_bits;
    pl.p_stage = packed_stage_bytes(bnn::TC_PLANE_CODES, a_bits, w_bits);
    pl.pstages = packed_stages(bnn::TC_PLANE_CODES, a_bits, w_bits);
    if (pl.pstages < 2) return BNN_ERR_UNSUPPORTED;
    bnn::GemmEpilogue e{};
    e.c_i32 = C_i32;
    e.ldc = ldc;
    e.c_f32 = C_f32;
    e.ldf = ldf;
    e.alpha = alpha;
    e.bits_words = packed_ld_words(N);
    const int64_t grid = std::min<int64_t>(tiles_m * tiles_n, sm_count());
    const size_t smem = (size_t)SMEM_FIXED + (size_t)pl.pstages * (size_t)pl.p_stage;
    bnn::xnor_gemm_tc_kernel<bnn::TC_PLANE_CODES><<<(unsigned)grid, THREADS, smem, as_cuda(stream)>>>(
        tmA, tmW, (int)M, (int)N, (int)K, (int)kw, (int)tiles_m, (int)tiles_n, e, pl);
    return launch_status();
}

bnn_status bnn_binary_bases_gemm(const uint32_t* H, int64_t ldh, int J, const uint32_t* B, int64_t ldb, int I,
                                 int64_t M, int64_t N, int64_t K, const float* beta, const float* alpha,
                                 int64_t lda_alpha, float* Y, int64_t ldy, bnn_stream_t stream) {
    using namespace bnn::tc;
    bnn_status st = check_gemm_dims(M, N, K);
    if (st != BNN_OK) return st;
    if (J < 1 || J > MAX_BASES || I < 1 || I > MAX_BASES) return BNN_ERR_INVALID_ARG;
    if (M * J > INT_MAX || N * I > INT_MAX) return BNN_ERR_INVALID_ARG;
    const int64_t kw = packed_ld_words(K);
    if ((st = check_packed_operand(H, ldh, kw)) != BNN_OK) return st;
    if ((st = check_packed_operand(B, ldb, kw)) != BNN_OK) return st;
    if (beta == nullptr || alpha == nullptr || Y == nullptr) return BNN_ERR_INVALID_ARG;
    if (lda_alpha < N || ldy < N) return BNN_ERR_INVALID_ARG;
    if (!aligned(beta, 4) || !aligned(alpha, 4) || !aligned(Y, 4)) return BNN_ERR_ALIGNMENT;
    if (M == 0 || N == 0) return BNN_OK;
    const int jp = pow2_at_least(J), ip = pow2_at_least(I);
    {
        // +1/-1 bases on the e2m1 kernel in CTA pairs: each CTA holds
        // 128 / jp output rows (x jp bases) and half of the tile's bn / ip
        // output columns (x ip bases).
        const int engine = g_gemm_engine.load(std::memory_order_relaxed);
        const int pairs = engine == BNN_GEMM_ENGINE_TENSOR_I8 ? -1 : gemm_f4_pairs_resident();
        const int rows_cta = bnn::f4::BM / jp;
        if (pairs > 0 && pairs < kNoPairs && M > rows_cta && f4_padded_k(K) <= bnn::f4::MAX_KP) {
            const int64_t tiles_m = ceil_div(M, (int64_t)2 * rows_cta);
            const int bn = f4_pair_tile_n(tiles_m, N, ip, pairs);
            CUtensorMap fA, fW, fC;
            std::memset(&fC, 0, sizeof(fC));
            constexpr int sbkw = bnn::f4::Cfg<true, bnn::TC_BASES>::S_BKW;   // two K atoms: 64-byte rows
            static_assert(sbkw == 16, "bases pairs stage two K atoms");
            if (!encode_plane_map(&fA, H, kw, J, M, ldh, jp, rows_cta, sbkw, CU_TENSOR_MAP_SWIZZLE_64B) ||
                !encode_plane_map(&fW, B, kw, I, N, ldb, ip, bn / 2 / ip, sbkw, CU_TENSOR_MAP_SWIZZLE_64B))
                return BNN_ERR_CUDA;
            bnn::TcPlanes pl{};
            pl.ja = jp;
            pl.jw = ip;
            pl.j_real = J;
            pl.i_real = I;
            pl.beta = beta;
            pl.alpha = alpha;
            pl.lda_alpha = lda_alpha;
            pl.y = Y;
            pl.ldy = ldy;
            return launch_f4_pairs<bnn::TC_BASES>(fA, fW, fC, fC, M, N, K, kw, bn, tiles_m, ceil_div(N, bn / ip), 0,
                                                  bnn::GemmEpilogue{}, pl, pairs, as_cuda(stream));
        }
    }
    const int rows_per_tile = BM / jp, cols_per_tile = BN / ip;
    CUtensorMap tmA, tmW;
    if (!encode_plane_map(&tmA, H, kw, J, M, ldh, jp, rows_per_tile) ||
        !encode_plane_map(&tmW, B, kw, I, N, ldb, ip, cols_per_tile))
        return BNN_ERR_CUDA;
    const int64_t tiles_m = ceil_div(M, rows_per_tile), tiles_n = ceil_div(N, cols_per_tile);
    if (tiles_m * tiles_n > INT_MAX) return BNN_ERR_INVALID_ARG;
    if (!gemm_tc_smem_configured()) return BNN_ERR_CUDA;
    bnn::TcPlanes pl{};
    pl.ja = jp;
    pl.jw = ip;
    pl.j_real = J;
    pl.i_real = I;
    pl.p_stage = P_STAGE;
    pl.pstages = PSTAGES;
    pl.beta = beta;
    pl.alpha = alpha;
    pl.lda_alpha = lda_alpha;
    pl.y = Y;
    pl.ldy = ldy;
    const int64_t grid = std::min<int64_t>(tiles_m * tiles_n, sm_count());
    bnn::xnor_gemm_tc_kernel<bnn::TC_BASES><<<(unsigned)grid, THREADS, SMEM_BYTES, as_cuda(stream)>>>(
        tmA, tmW, (int)M, (int)N, (int)K, (int)kw, (int)tiles_m, (int)tiles_n, bnn::GemmEpilogue{}, pl);
    return launch_status();
}

bnn_status bnn_binary_weight_gemv_i8(const uint32_t* W, int64_t ldw, const int8_t* x, int64_t N, int64_t K,
                                     const float* alpha, int alpha_per_row, const float* x_scale, int32_t* y_i32,
                                     float* y_f32, uint32_t flags, bnn_stream_t stream) {
    constexpr uint32_t kAll = BNN_GEMV_WEIGHTS_STATIC | BNN_GEMV_INPUTS_STATIC | BNN_GEMV_OUTPUT_FREE;
    if ((flags & ~kAll) != 0) return BNN_ERR_INVALID_ARG;
    if (x == nullptr || (y_i32 == nullptr && y_f32 == nullptr)) return BNN_ERR_INVALID_ARG;
    if (y_f32 != nullptr && alpha == nullptr) return BNN_ERR_INVALID_ARG;
    if (alpha_per_row != 0 && alpha_per_row != 1) return BNN_ERR_INVALID_ARG;
    if (N < 0 || K < 1 || N > INT_MAX / 2) return BNN_ERR_INVALID_ARG;
    const int64_t kw = packed_ld_words(K);
    bnn_status st = check_packed_operand(W, ldw, kw);
    if (st != BNN_OK) return st;
    if (kw > bnn::bwi8::MAX_KW) return BNN_ERR_UNSUPPORTED;
    if ((y_i32 != nullptr && !aligned(y_i32, 4)) || (y_f32 != nullptr && !aligned(y_f32, 4)) ||
        (alpha != nullptr && !aligned(alpha, 4)) || (x_scale != nullptr && !aligned(x_scale, 4)))
        return BNN_ERR_ALIGNMENT;
    if (N == 0) return BNN_OK;
    int64_t lpr = 1;
    while (lpr < 32 && lpr < kw / 4) lpr <<= 1;
    const int64_t rows_per_cta = (int64_t)bnn::bwi8::WARPS * bnn::bwi8::U * (32 / lpr);
    cudaLaunchConfig_t cfg{};
    cfg.gridDim = dim3((unsigned)ceil_div(N, rows_per_cta));
    cfg.blockDim = dim3(bnn::bwi8::THREADS);
    cfg.dynamicSmemBytes = (size_t)kw * 32;
    cfg.stream = as_cuda(stream);
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    attr[0].val.programmaticStreamSerializationAllowed = 1;
    cfg.attrs = attr;
    cfg.numAttrs = 1;
    const int prefetch = (flags & BNN_GEMV_WEIGHTS_STATIC) ? 1 : 0;
    const int xstatic = (flags & BNN_GEMV_INPUTS_STATIC) ? 1 : 0;
    const int dependent = flags == kAll ? 2 : 1;
    const cudaError_t e = cudaLaunchKernelEx(&cfg, bnn::bw_gemv_i8_kernel<bnn::bwi8::U>, W, ldw, x, (int)N, (int)K,
                                             (int)kw, alpha, alpha_per_row, x_scale, y_i32, y_f32, prefetch, xstatic,
                                             dependent);
    if (e != cudaSuccess) return BNN_ERR_CUDA;
    return launch_status();
}

int64_t bnn_ternary_ld_words(int64_t K) { return K < 1 ? -1 : bnn::ternary_ld_words(K); }

int64_t bnn_ternary_workspace_bytes(int64_t rows) { return rows < 0 ? -1 : 8 * (rows + 1); }

bnn_status bnn_ternary_pack(const void* w, bnn_dtype dt, int64_t rows, int64_t K, int64_t ld_w, double delta,
                            uint32_t* codes, int64_t ldq, float* gamma_out, void* workspace,
                            int64_t workspace_bytes, bnn_stream_t stream) {
    if (w == nullptr || codes == nullptr) return BNN_ERR_INVALID_ARG;
    if (rows < 0 || K < 1 || ld_w < K || std::isnan(delta)) return BNN_ERR_INVALID_ARG;
    if (dt != BNN_F32 && dt != BNN_BF16) return BNN_ERR_INVALID_ARG;
    if (rows > ((int64_t)1 << 40) / K) return BNN_ERR_INVALID_ARG;        // rows * K stays exact in fp64
    const int64_t nw = bnn::ternary_ld_words(K);
    if (ldq < nw) return BNN_ERR_INVALID_ARG;
    if ((ldq & 3) != 0 || !aligned(codes, 16)) return BNN_ERR_ALIGNMENT;
    const size_t es = dt == BNN_F32 ? 4 : 2;
    if (!aligned(w, es) || (gamma_out != nullptr && !aligned(gamma_out, 4))) return BNN_ERR_ALIGNMENT;
    const bool need_gamma = delta < 0.0 || gamma_out != nullptr;
    if (need_gamma) {
        if (workspace == nullptr || workspace_bytes < bnn_ternary_workspace_bytes(rows)) return BNN_ERR_INVALID_ARG;
        if (!aligned(workspace, 8)) return BNN_ERR_ALIGNMENT;
    }
    if (rows == 0) return BNN_OK;
    const bool vec_ok = aligned(w, 16) && ((ld_w * (int64_t)es) % 16 == 0);
    const int64_t blocks = ceil_div(rows, 8);
    if (blocks > INT_MAX) return BNN_ERR_INVALID_ARG;
    cudaStream_t s = as_cuda(stream);
    double* rowsum = static_cast<double*>(workspace);
    double* gamma_d = need_gamma ? rowsum + rows : nullptr;
    // Row sums (plain launch: ordered after all earlier work), then gamma and
    // the pack as programmatic dependents, each waiting for its predecessor
    // before reading what that one wrote.
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    attr[0].val.programmaticStreamSerializationAllowed = 1;
    cudaLaunchConfig_t cfg{};
    cfg.stream = s;
    cfg.attrs = attr;
    cfg.numAttrs = need_gamma ? 1 : 0;
    cudaError_t e = cudaSuccess;
    if (need_gamma) {
        if (dt == BNN_F32)
            bnn::ternary_abs_rowsum_kernel<float, 4><<<(unsigned)blocks, 256, 0, s>>>(
                static_cast<const float*>(w), rows, K, ld_w, vec_ok, rowsum);
        else
            bnn::ternary_abs_rowsum_kernel<__nv_bfloat16, 4><<<(unsigned)blocks, 256, 0, s>>>(
                static_cast<const __nv_bfloat16*>(w), rows, K, ld_w, vec_ok, rowsum);
        cfg.gridDim = dim3(1);
        cfg.blockDim = dim3(1024);
        e = cudaLaunchKernelEx(&cfg, bnn::ternary_gamma_kernel, (const double*)rowsum, rows, K, gamma_d, gamma_out);
        if (e != cudaSuccess) return BNN_ERR_CUDA;
    }
    const double* gsrc = delta < 0.0 ? gamma_d : nullptr;
    cfg.gridDim = dim3((unsigned)blocks);
    cfg.blockDim = dim3(256);
    if (dt == BNN_F32)
        e = cudaLaunchKernelEx(&cfg, bnn::pack_ternary_kernel<float, 4>, static_cast<const float*>(w), rows, K, ld_w,
                               vec_ok, gsrc, delta, codes, ldq);
    else
        e = cudaLaunchKernelEx(&cfg, bnn::pack_ternary_kernel<__nv_bfloat16, 4>,
                               static_cast<const __nv_bfloat16*>(w), rows, K, ld_w, vec_ok, gsrc, delta, codes, ldq);
    if (e != cudaSuccess) return BNN_ERR_CUDA;
    return launch_status();
}

// ---------------------------------------------------------------------------
// bnn_ternary_pack_noalloc: bnn_ternary_pack with its workspace in a
// library-owned device array instead of caller memory.
// ---------------------------------------------------------------------------
namespace {

// Row sums (one double per row) plus gamma: BNN_TERNARY_PACK_NOALLOC_MAX_ROWS
// + 1 doubles, about 2 MiB, held by every GPU that loads the library.
static __device__ __align__(256) double g_ternary_scratch[BNN_TERNARY_PACK_NOALLOC_MAX_ROWS + 1];

// The device address of g_ternary_scratch on the current device, looked up
// once per device (host code cannot use the symbol itself as a pointer) and
// kept for the life of the process; a cudaDeviceReset() after the look-up
// would leave the kept address stale (the header says not to do that).
void* ternary_scratch_address() {
    constexpr int kMaxDevices = 64;
    static std::atomic<void*> addr[kMaxDevices];
    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= kMaxDevices) return nullptr;
    void* p = addr[dev].load(std::memory_order_acquire);
    if (p != nullptr) return p;
    if (cudaGetSymbolAddress(&p, g_ternary_scratch) != cudaSuccess || p == nullptr) return nullptr;
    addr[dev].store(p, std::memory_order_release);
    return p;
}

}  // namespace

bnn_status bnn_ternary_pack_noalloc(const void* w, bnn_dtype dt, int64_t rows, int64_t K, int64_t ld_w, double delta,
                                    uint32_t* codes, int64_t ldq, float* gamma_out, bnn_stream_t stream) {
    if (rows > BNN_TERNARY_PACK_NOALLOC_MAX_ROWS) return BNN_ERR_UNSUPPORTED;
    if (rows < 0) return BNN_ERR_INVALID_ARG;
    void* scratch = ternary_scratch_address();
    if (scratch == nullptr) return BNN_ERR_CUDA;
    return bnn_ternary_pack(w, dt, rows, K, ld_w, delta, codes, ldq, gamma_out, scratch,
                            (int64_t)sizeof(g_ternary_scratch), stream);
}

bnn_status bnn_ternary_gemv_i8(const uint32_t* codes, int64_t ldq, const int8_t* x, int64_t N, int64_t K,
                               const float* w_scale, const float* x_scale, int32_t* y_i32, float* y_f32,
                               uint32_t flags, bnn_stream_t stream) {
    constexpr uint32_t kAll = BNN_GEMV_WEIGHTS_STATIC | BNN_GEMV_INPUTS_STATIC | BNN_GEMV_OUTPUT_FREE;
    if ((flags & ~kAll) != 0) return BNN_ERR_INVALID_ARG;
    if (codes == nullptr || x == nullptr || (y_i32 == nullptr && y_f32 == nullptr)) return BNN_ERR_INVALID_ARG;
    if (N < 0 || K < 1 || N > INT_MAX) return BNN_ERR_INVALID_ARG;
    const int64_t nw = bnn::ternary_ld_words(K);
    if (ldq < nw) return BNN_ERR_INVALID_ARG;
    if ((ldq & 3) != 0 || !aligned(codes, 16)) return BNN_ERR_ALIGNMENT;
    if ((y_i32 != nullptr && !aligned(y_i32, 4)) || (y_f32 != nullptr && !aligned(y_f32, 4)) ||
        (w_scale != nullptr && !aligned(w_scale, 4)) || (x_scale != nullptr && !aligned(x_scale, 4)))
        return BNN_ERR_ALIGNMENT;
    if (nw > bnn::tgv::MAX_WORDS) return BNN_ERR_UNSUPPORTED;
    if (N == 0) return BNN_OK;
    if (!ternary_gemv_smem_configured()) return BNN_ERR_CUDA;
    cudaLaunchConfig_t cfg{};
    cfg.blockDim = dim3(256);
    cfg.dynamicSmemBytes = (size_t)nw * 16;
    cfg.stream = as_cuda(stream);
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    attr[0].val.programmaticStreamSerializationAllowed = 1;
    cfg.attrs = attr;
    cfg.numAttrs = 1;
    const int prefetch = (flags & BNN_GEMV_WEIGHTS_STATIC) ? 1 : 0;
    const int xstatic = (flags & BNN_GEMV_INPUTS_STATIC) ? 1 : 0;
    const bool independent = flags == kAll;
    const int dependent = independent ? 2 : 1;
    const bool x_vec = aligned(x, 16);
    // Measured at the decode shape (K = 4096): 4 rows per warp for independent
    // steps (more, smaller blocks overlap consecutive launches), 8 for a
    // dependent chain.
    cudaError_t e;
    if (independent) {
        cfg.gridDim = dim3((unsigned)ceil_div(N, (int64_t)32));
        e = cudaLaunchKernelEx(&cfg, bnn::ternary_gemv_i8_kernel<256, 4, 2>, codes, ldq, x, (int)N, (int)K, (int)nw,
                               x_vec, w_scale, x_scale, y_i32, y_f32, prefetch, xstatic, dependent);
    } else {
        cfg.gridDim = dim3((unsigned)ceil_div(N, (int64_t)64));
        e = cudaLaunchKernelEx(&cfg, bnn::ternary_gemv_i8_kernel<256, 8, 2>, codes, ldq, x, (int)N, (int)K, (int)nw,
                               x_vec, w_scale, x_scale, y_i32, y_f32, prefetch, xstatic, dependent);
    }
    if (e != cudaSuccess) return BNN_ERR_CUDA;
    return launch_status();
}

bnn_status bnn_binary_linear_fused(const uint32_t* A, int64_t lda, const uint32_t* W, int64_t ldw, int64_t M,
                                   int64_t N, int64_t K, const bnn_epilogue* epi, void* out, int64_t ld_out,
                                   bnn_stream_t stream) {
    bnn_status st = check_gemm_dims(M, N, K);
    if (st != BNN_OK) return st;
    if (epi == nullptr || out == nullptr) return BNN_ERR_INVALID_ARG;
    const int64_t kw = packed_ld_words(K);
    if ((st = check_packed_operand(A, lda, kw)) != BNN_OK) return st;
    if ((st = check_packed_operand(W, ldw, kw)) != BNN_OK) return st;
    if (!aligned(out, 4)) return BNN_ERR_ALIGNMENT;
    bnn::GemmEpilogue ep{};
    switch (epi->mode) {
        case BNN_OUT_INT32:
            if (ld_out < N) return BNN_ERR_INVALID_ARG;
            ep.c_i32 = static_cast<int32_t*>(out);
            ep.ldc = ld_out;
            break;
        case BNN_OUT_SCALED_F32:
        case BNN_OUT_AFFINE_F32:
            if (ld_out < N || epi->alpha == nullptr) return BNN_ERR_INVALID_ARG;
            if (epi->mode == BNN_OUT_AFFINE_F32 && (epi->gamma == nullptr || epi->beta == nullptr))
                return BNN_ERR_INVALID_ARG;
            ep.c_f32 = static_cast<float*>(out);
            ep.ldf = ld_out;
            ep.alpha = epi->alpha;
            if (epi->mode == BNN_OUT_AFFINE_F32) {
                ep.gamma = epi->gamma;
                ep.beta = epi->beta;
            }
            break;
        case BNN_OUT_THRESHOLD_PACK:
            if (epi->popc_thresh == nullptr || epi->thresh_mode == nullptr) return BNN_ERR_INVALID_ARG;
            if (N > 0 && ld_out < packed_ld_words(N)) return BNN_ERR_INVALID_ARG;
            if ((ld_out & 3) != 0) return BNN_ERR_ALIGNMENT;
            ep.c_bits = static_cast<uint32_t*>(out);
            ep.ldb = ld_out;
            ep.thresh = epi->popc_thresh;
            ep.thresh_mode = epi->thresh_mode;
            break;
        default:
            return BNN_ERR_INVALID_ARG;
    }
    if (M == 0 || N == 0) return BNN_OK;
    return dispatch_gemm(A, lda, W, ldw, M, N, K, ep, as_cuda(stream));
}

// Geometry of the shifted-window convolution (stride 1): the virtual line of
// padded positions, its 128-position tiles, and the rows per A buffer that
// fit in shared memory next to the resident filters.  BNN_ERR_UNSUPPORTED
// when a buffer cannot hold one tile's window.
static bnn_status conv_window_plan(int64_t n, int64_t h, int64_t w, int64_t pad, int64_t cw, int64_t n_mma,
                                   bool f4, bnn::ConvWindow* g) {
    const int64_t Hp = h + 2 * pad, Wp = w + 2 * pad;
    const int64_t V = n * Hp * Wp;
    const int64_t halo = 2 * Wp + 2;
    if (V + 2 * halo + 256 > INT_MAX) return BNN_ERR_UNSUPPORTED;
    const int64_t tiles = ceil_div(V, (int64_t)bnn::ctw::BM);
    const int64_t fixed = bnn::conv_tcw_smem_bytes((int)cw, (int)n_mma, 0, f4);
    int64_t rb = (227 * 1024 - fixed) / (2 * bnn::conv_tcw_row_bytes((int)cw, f4));
    rb = std::min<int64_t>(rb, 16000) / 8 * 8;
    const int64_t grid = std::min<int64_t>(tiles, sm_count());
    const int64_t per_cta = ceil_div(tiles, grid);
    rb = std::min<int64_t>(rb, ceil_div(per_cta * bnn::ctw::BM + halo, (int64_t)8) * 8);
    if (rb < bnn::ctw::BM + halo) return BNN_ERR_UNSUPPORTED;
    g->n = (int)n; g->h = (int)h; g->w = (int)w; g->pad = (int)pad;
    g->Hp = (int)Hp; g->Wp = (int)Wp; g->oh = (int)(Hp - 2); g->ow = (int)(Wp - 2);
    g->V = (int)V; g->tiles = (int)tiles; g->rb = (int)rb; g->halo = (int)halo;
    g->seg_tiles = (int)((rb - halo) / bnn::ctw::BM);
    return BNN_OK;
}

bnn_status bnn_binary_conv3x3_fused(const uint32_t* X_nhwc_bits, int64_t n, int64_t c, int64_t h, int64_t w,
                                    const uint32_t* W_packed, int64_t ldw, int64_t cout, int64_t stride, int64_t pad,
                                    const bnn_epilogue* epi, void* out_nchw, bnn_stream_t stream) {
    if (X_nhwc_bits == nullptr || W_packed == nullptr || epi == nullptr || out_nchw == nullptr)
        return BNN_ERR_INVALID_ARG;
    if (n < 0 || c < 1 || h < 1 || w < 1 || cout < 0 || stride < 1 || pad < 0) return BNN_ERR_INVALID_ARG;
    if (h > INT_MAX / 4 || w > INT_MAX / 4 || c > INT_MAX / 16 || cout > INT_MAX || pad > 1024 || stride > 1024)
        return BNN_ERR_INVALID_ARG;
    const int64_t oh = (h + 2 * pad - 3) / stride + 1, ow = (w + 2 * pad - 3) / stride + 1;
    if (h + 2 * pad < 3 || w + 2 * pad < 3 || oh < 1 || ow < 1) return BNN_ERR_INVALID_ARG;
    const int64_t cw = (c + 31) / 32;
    if (ldw < 9 * cw) return BNN_ERR_INVALID_ARG;
    switch (epi->mode) {
        case BNN_OUT_INT32: break;
        case BNN_OUT_SCALED_F32:
            if (epi->alpha == nullptr) return BNN_ERR_INVALID_ARG;
            break;
        case BNN_OUT_AFFINE_F32:
            if (epi->alpha == nullptr || epi->gamma == nullptr || epi->beta == nullptr) return BNN_ERR_INVALID_ARG;
            break;
        case BNN_OUT_THRESHOLD_PACK: return BNN_ERR_UNSUPPORTED;
        default: return BNN_ERR_INVALID_ARG;
    }
    if (!aligned(X_nhwc_bits, 4) || !aligned(W_packed, 16) || !aligned(out_nchw, 4)) return BNN_ERR_ALIGNMENT;
    if (cw > 4) return BNN_ERR_UNSUPPORTED;
    const int64_t kwp = (9 * cw + 3) / 4 * 4;
    const size_t smem = (size_t)cout * kwp * 4 + (size_t)cout * 3 * 4;   // filters + alpha/gamma/beta
    if (smem > 200 * 1024) return BNN_ERR_UNSUPPORTED;
    if (n == 0 || cout == 0) return BNN_OK;
    const int64_t npix = n * oh * ow;
    bnn::ConvEpilogue ep{epi->mode, epi->alpha, epi->gamma, epi->beta, out_nchw};
    cudaStream_t s = as_cuda(stream);
    int engine = g_gemm_engine.load(std::memory_order_relaxed);
    // The window kernel runs on e2m1 operands where two words of K fit one
    // MMA (cw even) and the scale factors fit beside the two accumulators,
    // on int8 operands otherwise and under TENSOR_I8; the other tensor-core
    // kernel is int8 only.
    const bool i8_only = engine == BNN_GEMM_ENGINE_TENSOR_I8;
    if (i8_only) engine = BNN_GEMM_ENGINE_TENSOR;
    const int64_t n_mma = std::max<int64_t>(16, ceil_div(cout, (int64_t)16) * 16);
    // Tensor cores, stride 1: the shifted-window kernel, when the resident
    // filters and two A buffers of at least one tile's window fit.  AUTO takes
    // it where it was measured to win clearly (the ResNet-class layer: 64
    // filters, c = 64, 200k output pixels: 29 us against 62 us): at least 64
    // filters, c <= 64 and 16384 output pixels.
    const bool tc_window = engine == BNN_GEMM_ENGINE_TENSOR ||
                           (engine == BNN_GEMM_ENGINE_AUTO && cout >= 64 && cw <= 2 && npix >= 16384);
    if (tc_window && stride == 1 && cout <= bnn::ctc::MAX_N) {
        const bool f4 = !i8_only && cw % 2 == 0 && 2 * ceil_div(n_mma, (int64_t)32) * 32 + 32 <= 512;
        bnn::ConvWindow g{};
        const bnn_status st = conv_window_plan(n, h, w, pad, cw, n_mma, f4, &g);
        if (st == BNN_OK) {
            const int smem_w = bnn::conv_tcw_smem_bytes((int)cw, (int)n_mma, g.rb, f4);
            const uint32_t idesc = f4 ? bnn::f4::idesc((int)n_mma, 1)
                                      : (2u << 4) | (1u << 7) | (1u << 10) | ((uint32_t)(n_mma >> 3) << 17) |
                                            ((uint32_t)(bnn::ctw::BM >> 4) << 24);
            const int grid = std::min(g.tiles, sm_count());
            auto launch_w = [&](auto kern) -> bnn_status {
                if (cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, smem_w) != cudaSuccess)
                    return BNN_ERR_CUDA;
                // Programmatic dependent launch: the kernel's set-up overlaps
                // the previous kernel; its reads and stores wait for it.
                cudaLaunchConfig_t cfg{};
                cfg.gridDim = dim3((unsigned)grid);
                cfg.blockDim = dim3(bnn::ctw::THREADS);
                cfg.dynamicSmemBytes = (size_t)smem_w;
                cfg.stream = s;
                cudaLaunchAttribute attr[1];
                attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
                attr[0].val.programmaticStreamSerializationAllowed = 1;
                cfg.attrs = attr;
                cfg.numAttrs = 1;
                if (cudaLaunchKernelEx(&cfg, kern, X_nhwc_bits, (int)c, W_packed, ldw, (int)cout, (int)n_mma, idesc, g,
                                       ep) != cudaSuccess)
                    return BNN_ERR_CUDA;
                return launch_status();
            };
            if (f4) return cw == 2 ? launch_w(bnn::xnor_conv3x3_tcw_kernel<2, true>)
                                   : launch_w(bnn::xnor_conv3x3_tcw_kernel<4, true>);
            switch (cw) {
                case 1: return launch_w(bnn::xnor_conv3x3_tcw_kernel<1>);
                case 2: return launch_w(bnn::xnor_conv3x3_tcw_kernel<2>);
                case 3: return launch_w(bnn::xnor_conv3x3_tcw_kernel<3>);
                default: return launch_w(bnn::xnor_conv3x3_tcw_kernel<4>);
            }
        }
        if (st != BNN_ERR_UNSUPPORTED) return st;
    }
    // Tensor cores, other strides (when forced): per-pixel gather of up to 2
    // words per tap (c <= 64) and 256 filters, when the resident filters and
    // two A tiles fit in shared memory.
    if (engine == BNN_GEMM_ENGINE_TENSOR && cw <= 2 && cout <= bnn::ctc::MAX_N &&
        bnn::conv_tc_smem_bytes((int)cw, (int)n_mma) <= 227 * 1024) {
        const int smem_tc = bnn::conv_tc_smem_bytes((int)cw, (int)n_mma);
        const uint32_t idesc = (2u << 4) | (1u << 7) | (1u << 10) | ((uint32_t)(n_mma >> 3) << 17) |
                               ((uint32_t)(bnn::ctc::BM >> 4) << 24);
        const int64_t tiles = ceil_div(npix, (int64_t)bnn::ctc::BM);
        if (tiles > INT_MAX) return BNN_ERR_INVALID_ARG;
        const int64_t grid = std::min<int64_t>(tiles, sm_count());
        auto launch_tc = [&](auto kern) -> bnn_status {
            if (cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, smem_tc) != cudaSuccess)
                return BNN_ERR_CUDA;
            kern<<<(unsigned)grid, bnn::ctc::THREADS, smem_tc, s>>>(X_nhwc_bits, (int)n, (int)c, (int)h, (int)w,
                                                                    W_packed, ldw, (int)cout, (int)n_mma, idesc,
                                                                    (int)stride, (int)pad, (int)oh, (int)ow, ep);
            return launch_status();
        };
        return cw == 1 ? launch_tc(bnn::xnor_conv3x3_tc_kernel<1>) : launch_tc(bnn::xnor_conv3x3_tc_kernel<2>);
    }
    const int64_t tasks = ceil_div(npix, (int64_t)32) * ceil_div(cout, (int64_t)bnn::conv::FB);
    int sms = 148;
    {
        int dev = 0;
        if (cudaGetDevice(&dev) == cudaSuccess) cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);
    }
    // A whole number of CTAs per SM (the kernel strides over warp tasks), no
    // more CTAs than there are tasks.
    const int64_t blocks = std::max<int64_t>(
        1, std::min<int64_t>(ceil_div(tasks, bnn::conv::WARPS), (int64_t)sms * bnn::conv::CTAS_PER_SM));
#define BNN_CONV_CASE(CWV)                                                                                 \
    case CWV: {                                                                                            \
        auto kern = bnn::xnor_conv3x3_kernel<CWV>;                                                         \
        if (smem > 48 * 1024 &&                                                                            \
            cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem) != cudaSuccess) \
            return BNN_ERR_CUDA;                                                                           \
        kern<<<(unsigned)blocks, bnn::conv::THREADS, smem, s>>>(X_nhwc_bits, (int)n, (int)c, (int)h, (int)w,  \
                                                                W_packed, ldw, (int)cout, (int)stride,     \
                                                                (int)pad, (int)oh, (int)ow, ep);           \
        break;                                                                                             \
    }
    switch (cw) {
        BNN_CONV_CASE(1)
        BNN_CONV_CASE(2)
        BNN_CONV_CASE(3)
        BNN_CONV_CASE(4)
        default: return BNN_ERR_UNSUPPORTED;
    }
#undef BNN_CONV_CASE
    return launch_status();
}

bnn_status bnn_binary_conv1x1_fused(const uint32_t* X_nhwc_bits, int64_t n, int64_t c, int64_t h, int64_t w,
                                    const uint32_t* W_packed, int64_t ldw, int64_t cout, int64_t stride,
                                    const bnn_epilogue* epi, void* out_nchw, bnn_stream_t stream) {
    if (X_nhwc_bits == nullptr || W_packed == nullptr || epi == nullptr || out_nchw == nullptr)
        return BNN_ERR_INVALID_ARG;
    if (n < 0 || c < 1 || h < 1 || w < 1 || cout < 0 || stride < 1) return BNN_ERR_INVALID_ARG;
    if (h > INT_MAX / 4 || w > INT_MAX / 4 || c > INT_MAX / 16 || cout > INT_MAX || stride > 1024)
        return BNN_ERR_INVALID_ARG;
    const int64_t oh = (h - 1) / stride + 1, ow = (w - 1) / stride + 1;
    const int64_t cw = (c + 31) / 32;
    if (ldw < cw) return BNN_ERR_INVALID_ARG;
    switch (epi->mode) {
        case BNN_OUT_INT32: break;
        case BNN_OUT_SCALED_F32:
            if (epi->alpha == nullptr) return BNN_ERR_INVALID_ARG;
            break;
        case BNN_OUT_AFFINE_F32:
            if (epi->alpha == nullptr || epi->gamma == nullptr || epi->beta == nullptr) return BNN_ERR_INVALID_ARG;
            break;
        case BNN_OUT_THRESHOLD_PACK: return BNN_ERR_UNSUPPORTED;
        default: return BNN_ERR_INVALID_ARG;
    }
    if (!aligned(X_nhwc_bits, 4) || !aligned(W_packed, 4) || !aligned(out_nchw, 4)) return BNN_ERR_ALIGNMENT;
    if (cw > 16) return BNN_ERR_UNSUPPORTED;
    // The kernel instance's word capacity (1, 2, 4, 8, 16) fixes the filter
    // row stride in shared memory: bnn::xnor_conv1x1_kernel<cwp> uses
    // (cwp + 3) / 4 * 4 words per row.
    const int cwp = cw == 1 ? 1 : cw == 2 ? 2 : cw <= 4 ? 4 : cw <= 8 ? 8 : 16;
    const int64_t kwp = (cwp + 3) / 4 * 4;
    const size_t smem = (size_t)cout * kwp * 4 + (size_t)cout * 2 * 4;   // filters + gamma*alpha, beta
    if (smem > 200 * 1024) return BNN_ERR_UNSUPPORTED;
    if (n == 0 || cout == 0) return BNN_OK;
    const int64_t npix = n * oh * ow;
    bnn::ConvEpilogue ep{epi->mode, epi->alpha, epi->gamma, epi->beta, out_nchw};
    if (npix > INT_MAX - 4096 || cout * oh * ow > INT_MAX) return BNN_ERR_UNSUPPORTED;   // 32-bit pixel indices
    // One contiguous run of (pixel block, filter) units per warp: 4 CTAs per
    // SM, fewer when there are fewer than about 16 units per warp.
    const int64_t units = ceil_div(npix, (int64_t)(32 * bnn::c1x1::pixels_per_lane(cwp))) * cout;
    const int64_t blocks = std::max<int64_t>(
        1, std::min<int64_t>(ceil_div(units, (int64_t)bnn::conv::WARPS * 16),
                             (int64_t)sm_count() * bnn::conv::CTAS_PER_SM));
    cudaStream_t s = as_cuda(stream);
    auto launch = [&](auto kern) -> bnn_status {
        if (smem > 48 * 1024 &&
            cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem) != cudaSuccess)
            return BNN_ERR_CUDA;
        cudaLaunchConfig_t cfg{};
        cfg.gridDim = dim3((unsigned)blocks);
        cfg.blockDim = dim3(bnn::conv::THREADS);
        cfg.dynamicSmemBytes = smem;
        cfg.stream = s;
        cudaLaunchAttribute attr[1];
        attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
        attr[0].val.programmaticStreamSerializationAllowed = 1;
        cfg.attrs = attr;
        cfg.numAttrs = 1;
        if (cudaLaunchKernelEx(&cfg, kern, X_nhwc_bits, (int)n, (int)c, (int)h, (int)w, W_packed, ldw, (int)cout,
                               (int)stride, (int)oh, (int)ow, ep) != cudaSuccess)
            return BNN_ERR_CUDA;
        return launch_status();
    };
    auto by_mode = [&](auto k_int, auto k_scaled, auto k_affine) -> bnn_status {
        if (epi->mode == BNN_OUT_INT32) return launch(k_int);
        if (epi->mode == BNN_OUT_SCALED_F32) return launch(k_scaled);
        return launch(k_affine);
    };
#define BNN_C1_CASE(CWV)                                                                                      \
    case CWV:                                                                                                 \
        return by_mode(bnn::xnor_conv1x1_kernel<CWV, BNN_OUT_INT32>, bnn::xnor_conv1x1_kernel<CWV, BNN_OUT_SCALED_F32>, \
                       bnn::xnor_conv1x1_kernel<CWV, BNN_OUT_AFFINE_F32>);
    switch (cwp) {
        BNN_C1_CASE(1)
        BNN_C1_CASE(2)
        BNN_C1_CASE(4)
        BNN_C1_CASE(8)
        default: return by_mode(bnn::xnor_conv1x1_kernel<16, BNN_OUT_INT32>,
                                bnn::xnor_conv1x1_kernel<16, BNN_OUT_SCALED_F32>,
                                bnn::xnor_conv1x1_kernel<16, BNN_OUT_AFFINE_F32>);
    }
#undef BNN_C1_CASE
}

int64_t bnn_gemv_chain_workspace_words(void) { return bnn::chain::WORKSPACE_WORDS; }

bnn_status bnn_xnor_gemv_chain(const bnn_chain_layer* layers, int32_t L, const void* x, bnn_dtype x_dt, int64_t K,
                               int32_t* y_i32, float* y_f32, uint32_t* acts, int64_t ld_acts, uint32_t* workspace,
                               bnn_stream_t stream) {
    using namespace bnn::chain;
    if (layers == nullptr || L < 1 || L > MAX_LAYERS || x == nullptr || workspace == nullptr) return BNN_ERR_INVALID_ARG;
    if (x_dt != BNN_F32 && x_dt != BNN_BF16) return BNN_ERR_INVALID_ARG;
    if (y_i32 == nullptr && y_f32 == nullptr) return BNN_ERR_INVALID_ARG;
    if (K < 1) return BNN_ERR_INVALID_ARG;
    if (!aligned(workspace, 16) || !aligned(x, x_dt == BNN_F32 ? 4 : 2)) return BNN_ERR_ALIGNMENT;
    if (acts != nullptr && !aligned(acts, 4)) return BNN_ERR_ALIGNMENT;

    // every argument is checked before the first CUDA call
    int64_t k = K, hidden_kw = 0;
    for (int l = 0; l < L; ++l) {
        const bnn_chain_layer& c = layers[l];
        const bool hidden = l < L - 1;
        if (c.N < 1 || c.N > (int64_t(1) << 24)) return BNN_ERR_INVALID_ARG;
        if (k > (int64_t)MAX_KW * 32) return BNN_ERR_UNSUPPORTED;
        const bnn_status st = check_packed_operand(c.W, c.ldw, packed_ld_words(k));
        if (st != BNN_OK) return st;
        if (hidden && (c.popc_thresh == nullptr || c.thresh_mode == nullptr)) return BNN_ERR_INVALID_ARG;
        if (!hidden && y_f32 != nullptr && c.alpha == nullptr) return BNN_ERR_INVALID_ARG;
        if (hidden) hidden_kw = std::max(hidden_kw, packed_ld_words(c.N));
        k = c.N;
    }
    if (acts != nullptr && ld_acts < hidden_kw) return BNN_ERR_INVALID_ARG;

    auto kern = x_dt == BNN_F32 ? bnn::xnor_gemv_chain_kernel<float> : bnn::xnor_gemv_chain_kernel<__nv_bfloat16>;
    int per_sm = 0;
    if (cudaOccupancyMaxActiveBlocksPerMultiprocessor(&per_sm, kern, THREADS, 0) != cudaSuccess || per_sm < 1)
        return BNN_ERR_CUDA;
    const int64_t G = (int64_t)std::min(per_sm, 2) * sm_count();

    bnn::ChainArgs args{};
    k = K;
    for (int l = 0; l < L; ++l) {
        const bnn_chain_layer& c = layers[l];
        const int64_t kw = packed_ld_words(k);
        bnn::ChainLayer& ly = args.layer[l];
        ly.W = c.W;
        ly.thr = c.popc_thresh;
        ly.mode = c.thresh_mode;
        ly.alpha = c.alpha;
        ly.ldw = c.ldw;
        ly.N = (int)c.N;
        ly.K = (int)k;
        ly.kw = (int)kw;
        ly.rc = (int)ceil_div(c.N, G);
        ly.active = (int)ceil_div(c.N, ly.rc);
        const int nch = (int)(kw / 4);
        int lpr = 1;
        while (lpr < 32 && lpr < nch) lpr <<= 1;
        ly.lpr = lpr;
        ly.lpr_log2 = 0;
        while ((1 << ly.lpr_log2) < lpr) ++ly.lpr_log2;
        ly.np = (int)ceil_div(nch, lpr);                 // 1 .. 4 for kw <= 512
        k = c.N;
    }
    // Layer l zeroes the slots layer l + 2 writes; the zeroing blocks own rows
    // of layer l + 1 too (their adds there order the zeroes before layer l + 2).
    for (int l = 0; l < L; ++l) {
        bnn::ChainLayer& ly = args.layer[l];
        ly.zero_blocks = l + 2 <= L - 2 ? std::min(ly.active, args.layer[l + 1].active) : 0;
        ly.zero_words = ly.zero_blocks > 0 ? (int)ceil_div(args.layer[l + 2].N, 32) : 0;
        ly.zero_per = ly.zero_blocks > 0 ? (int)ceil_div(ly.zero_words, ly.zero_blocks) : 0;
    }
    args.x = x;
    args.y_i32 = y_i32;
    args.y_f32 = y_f32;
    args.acts = acts;
    args.ld_acts = ld_acts;
    args.slots = reinterpret_cast<unsigned long long*>(workspace + HEADER_WORDS);
    args.finished = workspace;
    args.L = L;
    args.x_vec = aligned(x, 16) ? 1 : 0;

    cudaLaunchConfig_t cfg{};
    cfg.gridDim = dim3((unsigned)G);
    cfg.blockDim = dim3(THREADS);
    cfg.dynamicSmemBytes = 0;
    cfg.stream = as_cuda(stream);
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeCooperative;
    attr[0].val.cooperative = 1;
    cfg.attrs = attr;
    cfg.numAttrs = 1;
    if (cudaLaunchKernelEx(&cfg, kern, args) != cudaSuccess) {
        (void)cudaGetLastError();
        return BNN_ERR_CUDA;
    }
    return launch_status();
}

}  // extern "C"
