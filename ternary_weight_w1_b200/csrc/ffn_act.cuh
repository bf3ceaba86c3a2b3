// The gated squared ReLU of the feed-forward chain when its gate and up
// projections run on the tensor cores (batches the fused GEMV launch does not
// take): h = (r * r) * up with r = max(gate, 0), from the two projections'
// bf16 outputs, in fp32. Both products are exact for bf16 operands (8-bit
// significands: r * r needs 16 bits, (r * r) * up 24), so h equals what the
// GEMV launch's epilogue writes for the same gate and up.
//
// Pages: "Microsoft Releases BitNet b1.58 2B4T", section "Under the Hood"
// (ReLU^2 in place of SwiGLU); "BitNet b1.58: The 1-Bit Paradigm Shift".
#pragma once

#include "common.cuh"

namespace bitlinear {
namespace ffn {

constexpr int THREADS = 256;

// n8: the element count / 8 (M * F with F a multiple of 128); gate, up and h
// 16-byte aligned.
__global__ void __launch_bounds__(THREADS)
relu2_glu_kernel(const uint16_t *__restrict__ gate, const uint16_t *__restrict__ up,
                 float *__restrict__ h, int64_t n8)
{
    pdl_launch_dependents();
    pdl_wait();                          // gate and up are the previous kernel's outputs
    const int64_t stride = static_cast<int64_t>(gridDim.x) * THREADS;
    for (int64_t i = static_cast<int64_t>(blockIdx.x) * THREADS + threadIdx.x; i < n8;
         i += stride) {
        const uint4 g = reinterpret_cast<const uint4 *>(gate)[i];
        const uint4 u = reinterpret_cast<const uint4 *>(up)[i];
        const uint32_t gw[4] = {g.x, g.y, g.z, g.w};
        const uint32_t uw[4] = {u.x, u.y, u.z, u.w};
        float out[8];
#pragma unroll
        for (int j = 0; j < 8; ++j) {
            const uint32_t gb = (j & 1) ? (gw[j >> 1] & 0xffff0000u) : (gw[j >> 1] << 16);
            const uint32_t ub = (j & 1) ? (uw[j >> 1] & 0xffff0000u) : (uw[j >> 1] << 16);
            const float gv = __uint_as_float(gb);
            const float r = gv > 0.0f ? gv : 0.0f;
            out[j] = __fmul_rn(__fmul_rn(r, r), __uint_as_float(ub));
        }
        float4 *dst = reinterpret_cast<float4 *>(h) + 2 * i;
        dst[0] = make_float4(out[0], out[1], out[2], out[3]);
        dst[1] = make_float4(out[4], out[5], out[6], out[7]);
    }
}

}  // namespace ffn
}  // namespace bitlinear
