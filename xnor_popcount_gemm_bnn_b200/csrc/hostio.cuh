// Copies between pinned host memory and the device made by the SMs' own
// loads and stores (the host buffers are mapped into the device's address
// space), for the small per-step vectors of a batch-1 product: a copy-engine
// transfer of a few KB costs several microseconds of setup and completion
// latency per call, while a kernel reads or writes the same bytes across
// PCIe in one round trip of whole 16-byte vectors and chains to its
// neighbours by programmatic dependent launch.  (Letting the product kernel
// store its outputs across PCIe itself, a few rows per warp, took twice as
// long per step as a separate copy of whole vectors.)
//
// copy16_kernel<SRC_EARLY> moves n16 16-byte vectors from src to dst.  The
// stores to dst always wait for the previous grid on the stream
// (griddepcontrol.wait).  SRC_EARLY: nothing still in flight writes src (an
// input that the host filled before the call), so the loads are issued
// before that wait and their PCIe latency overlaps the previous step; else
// (a device result) the loads follow the wait.
#pragma once

#include "common.cuh"

namespace bnn {
namespace hostio {
constexpr int THREADS = 256;
constexpr int VEC = 4;                 // 16-byte vectors per thread and pass
constexpr int MAX_BLOCKS = 16;
}  // namespace hostio

template <bool SRC_EARLY>
__global__ void __launch_bounds__(hostio::THREADS)
copy16_kernel(const uint4* src, uint4* dst, int64_t n16) {
    using namespace hostio;
    const int64_t stride = (int64_t)gridDim.x * THREADS;
    // The grid is a few resident blocks: the next kernel may be scheduled
    // now and waits for this one itself.
    grid_dependents_launch();
    if (!SRC_EARLY) grid_dependency_wait();
    for (int64_t base = (int64_t)blockIdx.x * THREADS + threadIdx.x; base < n16; base += stride * VEC) {
        uint4 v[VEC];
        #pragma unroll
        for (int k = 0; k < VEC; ++k) {
            const int64_t i = base + k * stride;
            if (i < n16) v[k] = src[i];
        }
        if (SRC_EARLY) grid_dependency_wait();
        #pragma unroll
        for (int k = 0; k < VEC; ++k) {
            const int64_t i = base + k * stride;
            if (i < n16) dst[i] = v[k];
        }
    }
    // A block without vectors still orders its exit after the previous grid.
    grid_dependency_wait();
}

}  // namespace bnn
