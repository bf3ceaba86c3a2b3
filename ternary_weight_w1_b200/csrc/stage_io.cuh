// Token staging for the host-buffer decode call (bitlinear_forward_grouped_host):
// copies the tokens of up to eight problems from host memory that the device
// can address (pinned and mapped into its address space) into the problems'
// device x buffers, so that a decode step needs no copy-engine transfer for
// its inputs. The copy is a plain kernel because a step's token is small
// (a few KiB to a few hundred KiB): the cost is the host-memory read latency,
// which the kernel takes before it waits for the previous kernel in the
// stream, not the bandwidth.
#pragma once

#include "common.cuh"

namespace bitlinear {
namespace stage {

constexpr int MAX_PIECES = 8;
constexpr int THREADS = 256;
constexpr int PER_THREAD = 4;       // 16-byte vectors a thread reads before the wait

struct Pieces {
    const uint4 *src;               // device-addressable host memory, pieces back to back
    uint4 *dst[MAX_PIECES];         // each piece's device buffer
    int end[MAX_PIECES];            // cumulative piece lengths in 16-byte vectors
    int count;
};

__device__ __forceinline__ void put(const Pieces &p, int e, const uint4 &v)
{
    int i = 0;
    while (i + 1 < p.count && e >= p.end[i])
        ++i;
    const int begin = i == 0 ? 0 : p.end[i - 1];
    p.dst[i][e - begin] = v;
}

__global__ void __launch_bounds__(THREADS) stage_tokens_kernel(const __grid_constant__ Pieces p)
{
    // The next kernel (the GEMV) may launch at once: its weight stream starts
    // while the tokens cross the bus, and it reads them only after this
    // kernel has completed.
    pdl_launch_dependents();
    const int total = p.end[p.count - 1];
    const int stride = static_cast<int>(gridDim.x) * THREADS;
    const int e0 = static_cast<int>(blockIdx.x) * THREADS + static_cast<int>(threadIdx.x);
    uint4 v[PER_THREAD];
#pragma unroll
    for (int i = 0; i < PER_THREAD; ++i) {
        const int e = e0 + i * stride;
        if (e < total)
            v[i] = p.src[e];
    }
    // The previous kernel in the stream (the last step's GEMV) may still be
    // reading the device buffers: write them only after it has completed.
    pdl_wait();
#pragma unroll
    for (int i = 0; i < PER_THREAD; ++i) {
        const int e = e0 + i * stride;
        if (e < total)
            put(p, e, v[i]);
    }
    for (int e = e0 + PER_THREAD * stride; e < total; e += stride)
        put(p, e, p.src[e]);
}

}  // namespace stage
}  // namespace bitlinear
