// Decode GEMV for small M: y = BitLinear(x) with the activation quantisation
// fused in the prologue and the packed ternary weights streamed from HBM once.
//
// Pages: "BitNet b1.58 2B4T Guide: Scaling Native 1-Bit LLMs", sections
// "8-Bit Activation Quantization: absmax Scaling" (prologue), "Matrix
// Multiplication as Pure Integer Addition" (contraction and rescale); the
// memory-wall framing of "BitNet b1.58: The 1-Bit Paradigm Shift" is why this
// kernel is organised around the weight bytes.
//
// Work split. Block b owns the contiguous rows [b*N/G, (b+1)*N/G) of W, which
// are one contiguous byte range of the packed matrix. A warp "unit" is 4 rows
// x 8 lanes: lane (rl, kl) loads 16 bytes (64 weights) of row rl at chunk
// q*8 + kl, so one warp-wide load touches four fully used 128-byte lines. The
// units of a block (pass-major, chunk-group-minor) are split evenly across its
// warps; each warp keeps DEPTH loads in flight per lane, and the first DEPTH
// are issued before the prologue so the weight stream overlaps it.
//
// Arithmetic. With codes c = W~ + 1 in {0,1,2}, masking a packed word with
// 0x03030303 << 2j leaves c * 4^j in each byte for the weights
// k = 16w + 4j .. 16w + 4j + 3. dp4a (unsigned codes x signed x~) into four
// plane accumulators, one per j, costs one AND and one dp4a per 4 weights
// and token; the plane sums are exact multiples of 4^j, so
//   sum c*x~ = a0 + (a1 >> 2) + (a2 >> 4) + (a3 >> 6)
// exactly, and acc = sum c*x~ - sum x~ (the row sum of x~ comes from the
// prologue). Lane partials are reduced over the 8 k-lanes by shuffles and added
// into per-row int32 shared-memory accumulators (integer, so the order of the
// atomic adds cannot change the result).
//
// x~ lives in shared memory "piece-major": for token m, chunk c (64 k's) and
// piece t (16 k's), bytes k = 64c + 16t .. +15 sit at m*K + (t*C + c)*16, so
// the eight k-lanes of a unit read eight consecutive 16-byte pieces (one
// conflict-free wavefront, broadcast over the four rows).
#pragma once

#include "common.cuh"

namespace bitlinear {
namespace gemv {

constexpr int THREADS = 256;
constexpr int WARPS = THREADS / 32;
constexpr int LK = 8;          // lanes across K in a unit
constexpr int LR = 32 / LK;    // rows in a unit

struct Params {
    const void *x;
    const uint8_t *packed;
    uint16_t *y;
    int32_t *acc_dbg;
    int8_t *xq_dbg;
    float *beta_dbg;
    int M, K, N;
    float gamma;
};

__host__ __device__ constexpr int smem_bytes(int MT, int K, int rows_cap)
{
    return MT * K + rows_cap * MT * 4 + 2 * MT * 4 + 2 * WARPS * 4;
}

__device__ __forceinline__ uint4 ldg_stream(const uint8_t *p)
{
    uint4 v;
    asm volatile("ld.global.nc.L1::no_allocate.v4.u32 {%0, %1, %2, %3}, [%4];"
                 : "=r"(v.x), "=r"(v.y), "=r"(v.z), "=r"(v.w)
                 : "l"(p));
    return v;
}

template <int MT, bool BF16, int DEPTH>
__global__ void __launch_bounds__(THREADS)
gemv_kernel(const Params p)
{
    extern __shared__ __align__(16) uint8_t smem[];
    const int K = p.K, M = p.M, N = p.N;
    const int C = K >> 6;                 // 16-byte chunks (64 weights) per row
    const int CG = (C + LK - 1) / LK;     // chunk groups per pass
    const int r0 = static_cast<int>((static_cast<int64_t>(blockIdx.x) * N) / gridDim.x);
    const int r1 = static_cast<int>((static_cast<int64_t>(blockIdx.x + 1) * N) / gridDim.x);
    const int nrows = r1 - r0;
    const int passes = (nrows + LR - 1) / LR;
    const int units = passes * CG;
    const int warp = threadIdx.x >> 5;
    const int lane = threadIdx.x & 31;
    const int rl = lane / LK;
    const int kl = lane % LK;
    const int u0 = static_cast<int>(static_cast<int64_t>(warp) * units / WARPS);
    const int u1 = static_cast<int>(static_cast<int64_t>(warp + 1) * units / WARPS);

    uint8_t *xq_sm = smem;
    int *acc_sm = reinterpret_cast<int *>(smem + MT * K);
    const int rows_cap = (N + gridDim.x - 1) / gridDim.x;
    float *beta_sm = reinterpret_cast<float *>(acc_sm + rows_cap * MT);
    int *rsum_sm = reinterpret_cast<int *>(beta_sm + MT);
    uint32_t *red_u = reinterpret_cast<uint32_t *>(rsum_sm + MT);
    int *red_i = reinterpret_cast<int *>(red_u + WARPS);

    const size_t row_bytes = static_cast<size_t>(K) >> 2;
    const uint8_t *wbase = p.packed + static_cast<size_t>(r0) * row_bytes;

    // ---- 1. start the weight stream (independent of x and of earlier kernels)
    int ld_p = u0 / CG, ld_q = u0 % CG;   // next unit to load
    auto load_next = [&]() -> uint4 {
        const int row = ld_p * LR + rl;
        const int chunk = ld_q * LK + kl;
        uint4 v = make_uint4(0u, 0u, 0u, 0u);
        if (row < nrows && chunk < C)
            v = ldg_stream(wbase + static_cast<size_t>(row) * row_bytes + chunk * 16);
        if (++ld_q == CG) {
            ld_q = 0;
            ++ld_p;
        }
        return v;
    };
    uint4 buf[DEPTH];
#pragma unroll
    for (int i = 0; i < DEPTH; ++i)
        buf[i] = (u0 + i < u1) ? load_next() : make_uint4(0u, 0u, 0u, 0u);

    for (int i = threadIdx.x; i < nrows * MT; i += THREADS)
        acc_sm[i] = 0;

    // ---- 2. prologue: absmax int8 quantisation of the M tokens
    pdl_wait();
    pdl_launch_dependents();
    for (int m = 0; m < M; ++m) {
        const void *row = static_cast<const char *>(p.x) +
                          static_cast<size_t>(m) * K * (BF16 ? 2 : 4);
        float amax = 0.0f;
        for (int e = threadIdx.x * 8; e < K; e += THREADS * 8) {
            float v[8];
            load8<BF16>(row, e, v);
#pragma unroll
            for (int i = 0; i < 8; ++i)
                amax = fmaxf(amax, fabsf(v[i]));
        }
        const float beta = fmaxf(block_max_nonneg<WARPS>(amax, red_u), 1e-5f);
        const float scale = __fdiv_rn(127.0f, beta);
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
            const int c = e >> 6, t = (e >> 4) & 3;
            *reinterpret_cast<uint2 *>(xq_sm + m * K + (t * C + c) * 16 + (e & 15)) =
                make_uint2(lo, hi);
            if (p.xq_dbg != nullptr && blockIdx.x == 0)
                *reinterpret_cast<uint2 *>(p.xq_dbg + static_cast<size_t>(m) * K + e) =
                    make_uint2(lo, hi);
        }
        const int total = block_sum_int<WARPS>(sum, red_i);
        if (threadIdx.x == 0) {
            beta_sm[m] = beta;
            rsum_sm[m] = total;
            if (p.beta_dbg != nullptr && blockIdx.x == 0)
                p.beta_dbg[m] = beta;
        }
    }
    __syncthreads();

    // ---- 3. stream the weights: dp4a over 4^j-scaled code planes
    int acc[MT][4];
#pragma unroll
    for (int m = 0; m < MT; ++m)
#pragma unroll
        for (int j = 0; j < 4; ++j)
            acc[m][j] = 0;

    int cur_p = u0 / CG, cur_q = u0 % CG;
    for (int base = u0; base < u1; base += DEPTH) {
#pragma unroll
        for (int i = 0; i < DEPTH; ++i) {
            const int u = base + i;
            if (u < u1) {
                const uint4 w = buf[i];
                if (u + DEPTH < u1)
                    buf[i] = load_next();
                const int chunk = cur_q * LK + kl;
                const int cx = chunk < C ? chunk : 0;   // any valid x~ piece; w is 0
                const uint32_t words[4] = {w.x, w.y, w.z, w.w};
                uint32_t mw[4][4];
#pragma unroll
                for (int t = 0; t < 4; ++t)
#pragma unroll
                    for (int j = 0; j < 4; ++j)
                        mw[t][j] = words[t] & (0x03030303u << (2 * j));
#pragma unroll
                for (int m = 0; m < MT; ++m) {
                    if (m < M) {
#pragma unroll
                        for (int t = 0; t < 4; ++t) {
                            const uint4 xv = *reinterpret_cast<const uint4 *>(
                                xq_sm + m * K + (t * C + cx) * 16);
                            acc[m][0] = dp4a_us(mw[t][0], xv.x, acc[m][0]);
                            acc[m][1] = dp4a_us(mw[t][1], xv.y, acc[m][1]);
                            acc[m][2] = dp4a_us(mw[t][2], xv.z, acc[m][2]);
                            acc[m][3] = dp4a_us(mw[t][3], xv.w, acc[m][3]);
                        }
                    }
                }
                const bool pass_end = (++cur_q == CG);
                if (pass_end || u + 1 == u1) {
                    const int row = cur_p * LR + rl;
#pragma unroll
                    for (int m = 0; m < MT; ++m) {
                        int v = acc[m][0] + (acc[m][1] >> 2) + (acc[m][2] >> 4) + (acc[m][3] >> 6);
                        v += __shfl_xor_sync(0xffffffffu, v, 1);
                        v += __shfl_xor_sync(0xffffffffu, v, 2);
                        v += __shfl_xor_sync(0xffffffffu, v, 4);
                        if (kl == 0 && row < nrows && m < M)
                            atomicAdd(&acc_sm[row * MT + m], v);
#pragma unroll
                        for (int j = 0; j < 4; ++j)
                            acc[m][j] = 0;
                    }
                    if (pass_end) {
                        cur_q = 0;
                        ++cur_p;
                    }
                }
            }
        }
    }
    __syncthreads();

    // ---- 4. epilogue: acc = sum c*x~ - sum x~, rescale, bf16
    for (int m = 0; m < M; ++m) {
        const float s = out_scale(beta_sm[m], p.gamma);
        const int rs = rsum_sm[m];
        for (int r = threadIdx.x; r < nrows; r += THREADS) {
            const int a = acc_sm[r * MT + m] - rs;
            const size_t o = static_cast<size_t>(m) * N + r0 + r;
            p.y[o] = rescale_bf16(a, s);
            if (p.acc_dbg != nullptr)
                p.acc_dbg[o] = a;
        }
    }
}

}  // namespace gemv
}  // namespace bitlinear
