// Per-token absmax int8 quantisation (page "BitNet b1.58 2B4T Guide: Scaling
// Native 1-Bit LLMs", section "8-Bit Activation Quantization: absmax Scaling";
// the listing's quantize_activations_int8 fixes the clamp(min=1e-5), the
// order x * (127 / beta) and ties-to-even rounding).
//
// One warp per token row, eight rows per block, no block barriers. Each lane
// keeps up to CACHE vectors of 8 activations in registers from the absmax
// pass, so rows of up to 32 * 8 * CACHE elements are read from memory once;
// longer rows are re-read in the second pass, from L1. The row sum of x~ is
// written for the tensor-core path, whose GEMM contracts the non-negative
// weight codes W~ + 1 (acc = sum x~ * code - sum x~).
#pragma once

#include "common.cuh"

namespace bitlinear {
namespace qa {

constexpr int THREADS = 256;
constexpr int ROWS_PER_BLOCK = THREADS / 32;

template <bool BF16, int CACHE>
__global__ void __launch_bounds__(THREADS)
quant_act_kernel(const void *__restrict__ x, int M, int K, int8_t *__restrict__ xq,
                 float *__restrict__ beta_out, int *__restrict__ rowsum_out)
{
    const int lane = threadIdx.x & 31;
    const int m = blockIdx.x * ROWS_PER_BLOCK + (threadIdx.x >> 5);
    pdl_wait();
    if (m >= M)
        return;
    const size_t elem = BF16 ? 2 : 4;
    const void *row = static_cast<const char *>(x) + static_cast<size_t>(m) * K * elem;
    const int nvec = K >> 3;

    Vec8<BF16> cache[CACHE];
    float amax = 0.0f;
#pragma unroll
    for (int i = 0; i < CACHE; ++i) {
        const int v = lane + 32 * i;
        if (v < nvec) {
            cache[i].load(row, v * 8);
#pragma unroll
            for (int j = 0; j < 8; ++j)
                amax = fmaxf(amax, fabsf(cache[i].get(j)));
        }
    }
    for (int v = lane + 32 * CACHE; v < nvec; v += 32) {
        Vec8<BF16> t;
        t.load(row, v * 8);
#pragma unroll
        for (int j = 0; j < 8; ++j)
            amax = fmaxf(amax, fabsf(t.get(j)));
    }
    const float beta =
        fmaxf(__uint_as_float(__reduce_max_sync(0xffffffffu, __float_as_uint(amax))), 1e-5f);
    const float scale = __fdiv_rn(127.0f, beta);

    int8_t *out = xq + static_cast<size_t>(m) * K;
    int sum = 0;
    auto quant_store = [&](const Vec8<BF16> &t, int v) {
        uint32_t lo = 0, hi = 0;
#pragma unroll
        for (int i = 0; i < 4; ++i) {
            const int q0 = quant1(t.get(i), scale);
            const int q1 = quant1(t.get(i + 4), scale);
            sum += q0 + q1;
            lo |= (static_cast<uint32_t>(q0) & 0xffu) << (8 * i);
            hi |= (static_cast<uint32_t>(q1) & 0xffu) << (8 * i);
        }
        *reinterpret_cast<uint2 *>(out + v * 8) = make_uint2(lo, hi);
    };
#pragma unroll
    for (int i = 0; i < CACHE; ++i) {
        const int v = lane + 32 * i;
        if (v < nvec)
            quant_store(cache[i], v);
    }
    for (int v = lane + 32 * CACHE; v < nvec; v += 32) {
        Vec8<BF16> t;
        t.load(row, v * 8);
        quant_store(t, v);
    }
    pdl_launch_dependents();
    sum = __reduce_add_sync(0xffffffffu, sum);
    if (lane == 0) {
        beta_out[m] = beta;
        if (rowsum_out != nullptr)
            rowsum_out[m] = sum;
    }
}

}  // namespace qa
}  // namespace bitlinear
