// Per-token absmax int8 quantisation (page "BitNet b1.58 2B4T Guide: Scaling
// Native 1-Bit LLMs", section "8-Bit Activation Quantization: absmax Scaling";
// the listing's quantize_activations_int8 fixes the clamp(min=1e-5), the
// order x * (127 / beta) and ties-to-even rounding).
//
// One block per token row. Pass 1 reduces max |x|; pass 2 re-reads the row
// (L1/L2 resident), writes x~ and, for the tensor-core path, the row sum of
// x~ that the GEMM epilogue needs (the GEMM contracts the non-negative weight
// codes W~ + 1, so acc = sum x~ * code - sum x~).
#pragma once

#include "common.cuh"

namespace bitlinear {
namespace qa {

constexpr int THREADS = 256;
constexpr int WARPS = THREADS / 32;

template <bool BF16>
__global__ void __launch_bounds__(THREADS)
quant_act_kernel(const void *__restrict__ x, int K, int8_t *__restrict__ xq,
                 float *__restrict__ beta_out, int *__restrict__ rowsum_out)
{
    __shared__ uint32_t red_u[WARPS];
    __shared__ int red_i[WARPS];
    const int m = blockIdx.x;
    const size_t elem = BF16 ? 2 : 4;
    const void *row = static_cast<const char *>(x) + static_cast<size_t>(m) * K * elem;

    pdl_wait();

    float amax = 0.0f;
    for (int e = threadIdx.x * 8; e < K; e += THREADS * 8) {
        float v[8];
        load8<BF16>(row, e, v);
#pragma unroll
        for (int i = 0; i < 8; ++i)
            amax = fmaxf(amax, fabsf(v[i]));
    }
    float beta = block_max_nonneg<WARPS>(amax, red_u);
    beta = fmaxf(beta, 1e-5f);
    const float scale = __fdiv_rn(127.0f, beta);

    int8_t *out = xq + static_cast<size_t>(m) * K;
    int sum = 0;
    for (int e = threadIdx.x * 8; e < K; e += THREADS * 8) {
        float v[8];
        load8<BF16>(row, e, v);
        uint32_t lo = 0, hi = 0;
#pragma unroll
        for (int i = 0; i < 4; ++i) {
            const int q0 = quant1(v[i], scale);
            const int q1 = quant1(v[i + 4], scale);
            sum += q0 + q1;
            lo |= (static_cast<uint32_t>(q0) & 0xffu) << (8 * i);
            hi |= (static_cast<uint32_t>(q1) & 0xffu) << (8 * i);
        }
        *reinterpret_cast<uint2 *>(out + e) = make_uint2(lo, hi);
    }
    pdl_launch_dependents();
    if (rowsum_out != nullptr) {
        const int total = block_sum_int<WARPS>(sum, red_i);
        if (threadIdx.x == 0)
            rowsum_out[m] = total;
    }
    if (threadIdx.x == 0)
        beta_out[m] = beta;
}

}  // namespace qa
}  // namespace bitlinear
