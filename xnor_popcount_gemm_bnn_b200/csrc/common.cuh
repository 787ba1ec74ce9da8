// Device-side helpers shared by the kernels of libbnn.so (sm_100a only).
//
// Packed layout (see include/bnn.h): bit j of word w of a row is element
// 32*w + j, 1 = -1 and 0 = +1; rows are padded with zero bits and zero words
// to a multiple of 4 words ("First Principles: Why Binary Ops Can Be
// Exponentially Faster", section 1: pad bits encode +1).
#pragma once

#include <cuda.h>
#include <cuda_bf16.h>
#include <cuda_runtime.h>
#include <stdint.h>

#include "bnn.h"

namespace bnn {

// ---------------------------------------------------------------------------
// device error flag: set by a kernel that gave up waiting on an asynchronous
// copy; read and cleared by bnn_device_error().  The first error wins.
// ---------------------------------------------------------------------------
__device__ int g_device_error = 0;

__device__ __forceinline__ void flag_device_error(int code) {
    atomicCAS(&g_device_error, 0, code);
}

// Give up on an mbarrier wait after this many nanoseconds (about one second).
constexpr unsigned long long kWaitTimeoutNs = 1000000000ull;

__device__ __forceinline__ unsigned long long globaltimer_ns() {
    unsigned long long t;
    asm volatile("mov.u64 %0, %%globaltimer;" : "=l"(t));
    return t;
}

__host__ __device__ constexpr int64_t packed_ld_words(int64_t K) {
    return ((K + 31) / 32 + 3) / 4 * 4;
}

// ---------------------------------------------------------------------------
// shared-memory address helpers
// ---------------------------------------------------------------------------
__device__ __forceinline__ uint32_t smem_u32(const void* p) {
    return static_cast<uint32_t>(__cvta_generic_to_shared(p));
}

// ---------------------------------------------------------------------------
// mbarrier (shared::cta)
// ---------------------------------------------------------------------------
__device__ __forceinline__ void mbar_init(uint64_t* bar, uint32_t count) {
    asm volatile("mbarrier.init.shared::cta.b64 [%0], %1;" ::"r"(smem_u32(bar)), "r"(count)
                 : "memory");
}

__device__ __forceinline__ void fence_mbarrier_init() {
    asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
}

__device__ __forceinline__ void fence_proxy_async_shared() {
    asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
}

__device__ __forceinline__ void mbar_arrive(uint64_t* bar) {
    asm volatile("mbarrier.arrive.shared::cta.b64 _, [%0];" ::"r"(smem_u32(bar)) : "memory");
}

__device__ __forceinline__ void mbar_arrive_expect_tx(uint64_t* bar, uint32_t bytes) {
    asm volatile("mbarrier.arrive.expect_tx.shared::cta.b64 _, [%0], %1;" ::"r"(smem_u32(bar)),
                 "r"(bytes)
                 : "memory");
}

__device__ __forceinline__ bool mbar_try_wait(uint64_t* bar, uint32_t parity) {
    uint32_t ok;
    asm volatile(
        "{\n\t.reg .pred p;\n\t"
        "mbarrier.try_wait.parity.shared::cta.b64 p, [%1], %2;\n\t"
        "selp.u32 %0, 1, 0, p;\n\t}"
        : "=r"(ok)
        : "r"(smem_u32(bar)), "r"(parity)
        : "memory");
    return ok != 0;
}

// Wait for the phase of parity `parity` to complete, for at most
// `timeout_ns` (about one second by default).  On time-out, flags
// BNN_ERR_DEVICE_TIMEOUT and returns false.
__device__ __forceinline__ bool mbar_wait_bounded(uint64_t* bar, uint32_t parity,
                                                  unsigned long long timeout_ns = kWaitTimeoutNs) {
    if (mbar_try_wait(bar, parity)) return true;
    const unsigned long long t0 = globaltimer_ns();
    while (true) {
        #pragma unroll 1
        for (int i = 0; i < 64; ++i)
            if (mbar_try_wait(bar, parity)) return true;
        if (globaltimer_ns() - t0 > timeout_ns) {
            flag_device_error(BNN_ERR_DEVICE_TIMEOUT);
            return false;
        }
    }
}

// Diagnostic: one thread waits on an mbarrier that nothing ever arrives on,
// so the bounded wait runs out after `timeout_ns`; records how it ended in
// g_selftest_result (1 = completed, 0 = ran out).
__device__ int g_selftest_result = -1;

__global__ void wait_timeout_selftest_kernel(unsigned long long timeout_ns) {
    __shared__ uint64_t bar;
    if (threadIdx.x == 0) {
        mbar_init(&bar, 1);
        fence_mbarrier_init();
    }
    __syncthreads();
    if (threadIdx.x == 0) g_selftest_result = mbar_wait_bounded(&bar, 0, timeout_ns) ? 1 : 0;
}

// ---------------------------------------------------------------------------
// TMA: 2-D tiled bulk tensor load global -> shared, completion on an mbarrier.
// No multicast.
// ---------------------------------------------------------------------------
__device__ __forceinline__ void tma_load_2d(void* smem_dst, const CUtensorMap* map, int32_t x,
                                            int32_t y, uint64_t* bar) {
    asm volatile(
        "cp.async.bulk.tensor.2d.shared::cluster.global.mbarrier::complete_tx::bytes"
        " [%0], [%1, {%2, %3}], [%4];" ::"r"(smem_u32(smem_dst)),
        "l"(reinterpret_cast<uint64_t>(map)), "r"(x), "r"(y), "r"(smem_u32(bar))
        : "memory");
}

// 3-D variant: coordinates (x, y, z) = (word, plane, row) for operands whose
// rows carry several bit planes.  No multicast.
__device__ __forceinline__ void tma_load_3d(void* smem_dst, const CUtensorMap* map, int32_t x, int32_t y,
                                            int32_t z, uint64_t* bar) {
    asm volatile(
        "cp.async.bulk.tensor.3d.shared::cluster.global.mbarrier::complete_tx::bytes"
        " [%0], [%1, {%2, %3, %4}], [%5];" ::"r"(smem_u32(smem_dst)),
        "l"(reinterpret_cast<uint64_t>(map)), "r"(x), "r"(y), "r"(z), "r"(smem_u32(bar))
        : "memory");
}

__device__ __forceinline__ void prefetch_tensormap(const CUtensorMap* map) {
    asm volatile("prefetch.tensormap [%0];" ::"l"(reinterpret_cast<uint64_t>(map)) : "memory");
}

// ---------------------------------------------------------------------------
// global loads
// ---------------------------------------------------------------------------
// 16-byte read-only load that does not allocate in L1 (streamed data).
__device__ __forceinline__ uint4 ldg_stream_v4(const void* p) {
    uint4 v;
    asm volatile("ld.global.nc.L1::no_allocate.v4.u32 {%0, %1, %2, %3}, [%4];"
                 : "=r"(v.x), "=r"(v.y), "=r"(v.z), "=r"(v.w)
                 : "l"(p));
    return v;
}

__device__ __forceinline__ uint32_t popc_xor4(uint4 a, uint4 b) {
    return __popc(a.x ^ b.x) + __popc(a.y ^ b.y) + __popc(a.z ^ b.z) + __popc(a.w ^ b.w);
}

// Programmatic dependent launch controls (no-ops when the grid was not
// launched with the programmatic-serialisation attribute).
__device__ __forceinline__ void grid_dependency_wait() {
    asm volatile("griddepcontrol.wait;" ::: "memory");
}
__device__ __forceinline__ void grid_dependents_launch() {
    asm volatile("griddepcontrol.launch_dependents;" ::: "memory");
}
// End of a launch that depends on nothing still in flight: its completion
// must still imply the previous grid's, so that stream order stays
// transitive for later work.  A grid completes when its last block exits, so
// it is enough that one block (block 0) waits for the previous grid before
// exiting; the other blocks leave as soon as their work is stored and free
// their slots for the launches behind them.
__device__ __forceinline__ void exit_after_previous_grid() {
    if (blockIdx.x == 0) grid_dependency_wait();
}

// Real-valued element access for the two input dtypes.
__device__ __forceinline__ float to_float(float v) { return v; }
__device__ __forceinline__ float to_float(__nv_bfloat16 v) { return __bfloat162float(v); }

// sign() of "Extreme Quantization: Binary, Ternary & 1-bit LLMs", Notation:
// -1 (bit 1) exactly when x < 0.  An IEEE compare without flush-to-zero, so
// -0.0 and NaN give +1 and negative denormals give -1.
__device__ __forceinline__ uint32_t neg_bit(float v) { return v < 0.0f ? 1u : 0u; }

}  // namespace bnn
