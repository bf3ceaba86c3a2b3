// Per-token absmax int8 quantisation (page "BitNet b1.58 2B4T Guide: Scaling
// Native 1-Bit LLMs", section "8-Bit Activation Quantization: absmax Scaling";
// the listing's quantize_activations_int8 fixes the clamp(min=1e-5), the
// order x * (127 / beta) and ties-to-even rounding).
//
// WPR warps per token row (one for rows up to a few thousand elements, eight
// for long rows), 256 threads per block. Each lane keeps CACHE vectors of 8
// activations in registers from the absmax pass, so a row is read from
// memory once when 32 * WPR * 8 * CACHE covers it; anything beyond is
// re-read in the second pass, four vectors in flight per lane. A grouped
// variant quantises the rows of several problems in one launch (each with
// its own gains when it normalises).
//
// With NORM the row is RMS-normalised first, as the listing's BitLinear does
// with its nn.RMSNorm member before quantising: a first pass sums the squares
// in double (exact products; the butterfly and the fixed warp order make the
// sum the same in every block), r = 1 / sqrt(mean + eps) in IEEE fp32, and
// the absmax and quantisation passes work on (x * r) * g with the channel
// gains g read as they are needed. The row sum
// of x~ is written for the tensor-core path, whose GEMM contracts the
// non-negative weight codes W~ + 1 (acc = sum x~ * code - sum x~). Block 0
// also clears the GEMM's inter-block flag words when asked to. Prefill
// batches take a variant that stages whole rows in shared memory with bulk
// copies (quant_act_staged_kernel), so that one wave of blocks covers them.
#pragma once

#include "common.cuh"

namespace bitlinear {
namespace qa {

constexpr int THREADS = 256;
constexpr int WARPS = THREADS / 32;

template <int WPR>
__host__ __device__ constexpr int rows_per_block() { return WARPS / WPR; }

// Quantises token row m of one problem (warp `part` of the WPR warps that
// share the row); rows past M take part in the block barriers only. With
// NORM, gain [K] and eps define the RMS normalisation applied first.
template <bool BF16, int CACHE, int WPR, bool NORM>
__device__ __forceinline__ void quant_row(const void *__restrict__ x, int M, int K,
                                          int8_t *__restrict__ xq, float *__restrict__ beta_out,
                                          int *__restrict__ rowsum_out,
                                          const float *__restrict__ gain, float eps, int m,
                                          int part)
{
    static_assert(WARPS % WPR == 0, "warps per row");
    constexpr int STRIDE = 32 * WPR;              // vectors between a lane's vectors
    __shared__ uint32_t red_max[WARPS];
    __shared__ int red_sum[WARPS];
    const int warp = threadIdx.x >> 5;
    const int lane = threadIdx.x & 31;
    const bool active = m < M;
    if (WPR == 1 && !active)
        return;
    const size_t elem = BF16 ? 2 : 4;
    const void *row = static_cast<const char *>(x) +
                      static_cast<size_t>(active ? m : 0) * K * elem;
    const int nvec = active ? (K >> 3) : 0;
    const int v0 = part * 32 + lane;

    Vec8<BF16> cache[CACHE];
    float amax = 0.0f;
    float r = 1.0f;                               // NORM: 1 / rms of the row
    if constexpr (!NORM) {
        // bf16: the largest 15-bit magnitude field, two per word (for finite
        // values that order is the order of |x|), widened at the end
        uint32_t mb = 0;
        auto take = [&](const Vec8<BF16> &t) {
            if constexpr (BF16) {
#pragma unroll
                for (int j = 0; j < 4; ++j)
                    mb = max_u16x2(mb, t.w[j] & 0x7fff7fffu);
            } else {
#pragma unroll
                for (int j = 0; j < 8; ++j)
                    amax = fmaxf(amax, fabsf(t.get(j)));
            }
        };
#pragma unroll
        for (int i = 0; i < CACHE; ++i) {
            const int v = v0 + STRIDE * i;
            if (v < nvec) {
                cache[i].load(row, v * 8);
                take(cache[i]);
            }
        }
        for (int vb = v0 + STRIDE * CACHE; vb < nvec; vb += 4 * STRIDE) {
            Vec8<BF16> t[4];
#pragma unroll
            for (int u = 0; u < 4; ++u)
                if (vb + u * STRIDE < nvec)
                    t[u].load(row, (vb + u * STRIDE) * 8);
#pragma unroll
            for (int u = 0; u < 4; ++u)
                if (vb + u * STRIDE < nvec)
                    take(t[u]);
        }
        if constexpr (BF16)
            amax = __uint_as_float(max(mb & 0xffffu, mb >> 16) << 16);
    } else {
        // sum of squares (each product exact in double)
        double ss = 0.0;
#pragma unroll
        for (int i = 0; i < CACHE; ++i) {
            const int v = v0 + STRIDE * i;
            if (v < nvec) {
                cache[i].load(row, v * 8);
#pragma unroll
                for (int j = 0; j < 8; ++j) {
                    const double d = cache[i].get(j);
                    ss = __fma_rn(d, d, ss);
                }
            }
        }
        for (int vb = v0 + STRIDE * CACHE; vb < nvec; vb += STRIDE) {
            Vec8<BF16> t;
            t.load(row, vb * 8);
#pragma unroll
            for (int j = 0; j < 8; ++j) {
                const double d = t.get(j);
                ss = __fma_rn(d, d, ss);
            }
        }
        ss = warp_sum_f64(ss);
        if constexpr (WPR > 1) {
            __shared__ double red_ss[WARPS];
            if (lane == 0)
                red_ss[warp] = ss;
            __syncthreads();
            const int w0 = warp - part;
            ss = red_ss[w0];
#pragma unroll
            for (int w = 1; w < WPR; ++w)
                ss = __dadd_rn(ss, red_ss[w0 + w]);
        }
        r = rms_scale(ss, K, eps);
        // absmax of the normalised row
#pragma unroll
        for (int i = 0; i < CACHE; ++i) {
            const int v = v0 + STRIDE * i;
            if (v < nvec) {
                float g[8];
                load8<false>(gain, v * 8, g);
#pragma unroll
                for (int j = 0; j < 8; ++j)
                    amax = fmaxf(amax, fabsf(norm1(cache[i].get(j), r, g[j])));
            }
        }
        for (int vb = v0 + STRIDE * CACHE; vb < nvec; vb += STRIDE) {
            Vec8<BF16> t;
            float g[8];
            t.load(row, vb * 8);
            load8<false>(gain, vb * 8, g);
#pragma unroll
            for (int j = 0; j < 8; ++j)
                amax = fmaxf(amax, fabsf(norm1(t.get(j), r, g[j])));
        }
    }
    uint32_t umax = __reduce_max_sync(0xffffffffu, __float_as_uint(amax));
    if constexpr (WPR > 1) {
        if (lane == 0)
            red_max[warp] = umax;
        __syncthreads();
        const int w0 = warp - part;
        umax = red_max[w0];
#pragma unroll
        for (int w = 1; w < WPR; ++w)
            umax = max(umax, red_max[w0 + w]);
    }
    const float beta = fmaxf(__uint_as_float(umax), 1e-5f);
    const float scale = __fdiv_rn(127.0f, beta);

    int8_t *out = xq + static_cast<size_t>(active ? m : 0) * K;
    int sum = 0;
    auto quant_store = [&](const Vec8<BF16> &t, int v) {
        float g[8];
        if constexpr (NORM)
            load8<false>(gain, v * 8, g);
        uint32_t lo = 0, hi = 0;
#pragma unroll
        for (int i = 0; i < 4; ++i) {
            float a = t.get(i), b = t.get(i + 4);
            if constexpr (NORM) {
                a = norm1(a, r, g[i]);
                b = norm1(b, r, g[i + 4]);
            }
            const int q0 = quant1(a, scale);
            const int q1 = quant1(b, scale);
            sum += q0 + q1;
            lo |= (static_cast<uint32_t>(q0) & 0xffu) << (8 * i);
            hi |= (static_cast<uint32_t>(q1) & 0xffu) << (8 * i);
        }
        *reinterpret_cast<uint2 *>(out + v * 8) = make_uint2(lo, hi);
    };
#pragma unroll
    for (int i = 0; i < CACHE; ++i) {
        const int v = v0 + STRIDE * i;
        if (v < nvec)
            quant_store(cache[i], v);
    }
    for (int vb = v0 + STRIDE * CACHE; vb < nvec; vb += 4 * STRIDE) {
        Vec8<BF16> t[4];
#pragma unroll
        for (int u = 0; u < 4; ++u)
            if (vb + u * STRIDE < nvec)
                t[u].load(row, (vb + u * STRIDE) * 8);
#pragma unroll
        for (int u = 0; u < 4; ++u)
            if (vb + u * STRIDE < nvec)
                quant_store(t[u], vb + u * STRIDE);
    }
    pdl_launch_dependents();
    sum = __reduce_add_sync(0xffffffffu, sum);
    if constexpr (WPR > 1) {
        if (lane == 0)
            red_sum[warp] = sum;
        __syncthreads();
        const int w0 = warp - part;
        sum = 0;
#pragma unroll
        for (int w = 0; w < WPR; ++w)
            sum += red_sum[w0 + w];
    }
    if (active && part == 0 && lane == 0) {
        beta_out[m] = beta;
        if (rowsum_out != nullptr)
            rowsum_out[m] = sum;
    }
}

template <bool BF16, int CACHE, int WPR, bool NORM>
__global__ void __launch_bounds__(THREADS)
quant_act_kernel(const void *__restrict__ x, int M, int K, int8_t *__restrict__ xq,
                 float *__restrict__ beta_out, int *__restrict__ rowsum_out,
                 int *__restrict__ clear, int n_clear, const float *__restrict__ gain, float eps)
{
    const int warp = threadIdx.x >> 5;
    const int m = blockIdx.x * rows_per_block<WPR>() + warp / WPR;
    pdl_wait();
    // The GEMM that follows uses these words as inter-block flags; they are
    // cleared here, after every earlier grid in the stream has finished.
    if (clear != nullptr && blockIdx.x == 0)
        for (int i = threadIdx.x; i < n_clear; i += THREADS)
            clear[i] = 0;
    quant_row<BF16, CACHE, WPR, NORM>(x, M, K, xq, beta_out, rowsum_out, gain, eps, m,
                                      warp % WPR);
}

// Rows staged in shared memory, for prefill batches: thread 0 brings the
// block's R whole rows into shared memory with one bulk copy per row, all
// completing on one mbarrier, so a block keeps R rows in flight without
// holding them in registers and one wave of blocks covers the batch. Warp w
// then quantises rows w, w + WARPS, ... from shared memory in two passes
// (absmax, then quantise and store; with NORM a sum-of-squares pass first)
// with quant_row's arithmetic for one warp per row, so x~, beta and the row
// sums are the same bits as quant_row with one warp per row gives. A wait
// that gives up records the fault and the block writes nothing.
template <bool BF16, bool NORM>
__global__ void __launch_bounds__(THREADS)
quant_act_staged_kernel(const void *__restrict__ x, int M, int K, int rpb,
                        int8_t *__restrict__ xq, float *__restrict__ beta_out,
                        int *__restrict__ rowsum_out, int *__restrict__ clear, int n_clear,
                        const float *__restrict__ gain, float eps, uint64_t limit_ns)
{
    extern __shared__ __align__(128) uint8_t rows_sm[];
    __shared__ __align__(8) uint64_t bar_sm;
    __shared__ int abort_sm;
    const int warp = threadIdx.x >> 5;
    const int lane = threadIdx.x & 31;
    const uint32_t bar = smem_u32(&bar_sm);
    const int m0 = blockIdx.x * rpb;
    const int rows = min(rpb, M - m0);
    const uint32_t row_bytes = static_cast<uint32_t>(K) * (BF16 ? 2u : 4u);
    if (threadIdx.x == 0) {
        mbar_init(bar, 1);
        abort_sm = 0;
        fence_barrier_init();
    }
    __syncthreads();
    pdl_wait();
    // The GEMM that follows uses these words as inter-block flags.
    if (clear != nullptr && blockIdx.x == 0)
        for (int i = threadIdx.x; i < n_clear; i += THREADS)
            clear[i] = 0;
    if (threadIdx.x == 0) {
        mbar_arrive_expect_tx(bar, row_bytes * static_cast<uint32_t>(rows));
        for (int r = 0; r < rows; ++r)
            bulk_g2s(smem_u32(rows_sm) + static_cast<uint32_t>(r) * row_bytes,
                     static_cast<const char *>(x) + static_cast<size_t>(m0 + r) * row_bytes,
                     row_bytes, bar);
    }
    // every lane of a warp takes the same verdict, so the warp's reductions
    // below run with all its lanes or with none
    const bool ok =
        __all_sync(0xffffffffu, mbar_wait_bounded(bar, 0u, &abort_sm, limit_ns)) != 0;
    pdl_launch_dependents();
    if (ok) {
        const int nvec = K >> 3;
        constexpr int VB = BF16 ? 16 : 32;              // bytes per vector of 8
        for (int r = warp; r < rows; r += WARPS) {
            const uint8_t *row = rows_sm + static_cast<size_t>(r) * row_bytes;
            auto vec = [&](int v) {
                Vec8<BF16> t;
                const uint4 *src = reinterpret_cast<const uint4 *>(row + static_cast<size_t>(v) * VB);
#pragma unroll
                for (int i = 0; i < Vec8<BF16>::WORDS / 4; ++i) {
                    const uint4 a = src[i];
                    t.w[4 * i] = a.x; t.w[4 * i + 1] = a.y; t.w[4 * i + 2] = a.z; t.w[4 * i + 3] = a.w;
                }
                return t;
            };
            float amax = 0.0f;
            float rn = 1.0f;                            // NORM: 1 / rms of the row
            if constexpr (NORM) {
                double ss = 0.0;
                for (int v = lane; v < nvec; v += 32) {
                    const Vec8<BF16> t = vec(v);
#pragma unroll
                    for (int j = 0; j < 8; ++j) {
                        const double d = t.get(j);
                        ss = __fma_rn(d, d, ss);
                    }
                }
                rn = rms_scale(warp_sum_f64(ss), K, eps);
                for (int v = lane; v < nvec; v += 32) {
                    const Vec8<BF16> t = vec(v);
                    float g[8];
                    load8<false>(gain, v * 8, g);
#pragma unroll
                    for (int j = 0; j < 8; ++j)
                        amax = fmaxf(amax, fabsf(norm1(t.get(j), rn, g[j])));
                }
            } else if constexpr (BF16) {
                uint32_t mb = 0;
                for (int v = lane; v < nvec; v += 32) {
                    const Vec8<BF16> t = vec(v);
#pragma unroll
                    for (int j = 0; j < 4; ++j)
                        mb = max_u16x2(mb, t.w[j] & 0x7fff7fffu);
                }
                amax = __uint_as_float(max(mb & 0xffffu, mb >> 16) << 16);
            } else {
                for (int v = lane; v < nvec; v += 32) {
                    const Vec8<BF16> t = vec(v);
#pragma unroll
                    for (int j = 0; j < 8; ++j)
                        amax = fmaxf(amax, fabsf(t.get(j)));
                }
            }
            const uint32_t umax = __reduce_max_sync(0xffffffffu, __float_as_uint(amax));
            const float beta = fmaxf(__uint_as_float(umax), 1e-5f);
            const float scale = __fdiv_rn(127.0f, beta);
            const int m = m0 + r;
            int8_t *out = xq + static_cast<size_t>(m) * K;
            int sum = 0;
            for (int v = lane; v < nvec; v += 32) {
                const Vec8<BF16> t = vec(v);
                float g[8];
                if constexpr (NORM)
                    load8<false>(gain, v * 8, g);
                uint32_t lo = 0, hi = 0;
#pragma unroll
                for (int i = 0; i < 4; ++i) {
                    float a = t.get(i), b = t.get(i + 4);
                    if constexpr (NORM) {
                        a = norm1(a, rn, g[i]);
                        b = norm1(b, rn, g[i + 4]);
                    }
                    const int q0 = quant1(a, scale);
                    const int q1 = quant1(b, scale);
                    sum += q0 + q1;
                    lo |= (static_cast<uint32_t>(q0) & 0xffu) << (8 * i);
                    hi |= (static_cast<uint32_t>(q1) & 0xffu) << (8 * i);
                }
                *reinterpret_cast<uint2 *>(out + v * 8) = make_uint2(lo, hi);
            }
            sum = __reduce_add_sync(0xffffffffu, sum);
            if (lane == 0) {
                beta_out[m] = beta;
                if (rowsum_out != nullptr)
                    rowsum_out[m] = sum;
            }
        }
    } else if (threadIdx.x == 0) {
        // no copy may land after the block has exited
        drain_wait(bar, 0u, limit_ns);
    }
}

// Several problems' token rows in one launch (WPR warps per row): block b
// belongs to the problem whose block range [first_block, next first_block)
// holds it.
constexpr int MAX_PROBLEMS = 8;

struct GroupRows {
    const void *x;
    int8_t *xq;
    float *beta;
    int *rowsum;
    int M, K;
    int first_block;
    const float *gain;      // [K] RMS-normalisation gains (NORM launches only)
    float eps;
};

struct GroupParams {
    GroupRows prob[MAX_PROBLEMS];
    int count;
    int *clear;
    int n_clear;
};

template <bool BF16, int CACHE, int WPR, bool NORM>
__global__ void __launch_bounds__(THREADS)
quant_act_grouped_kernel(const __grid_constant__ GroupParams g)
{
    int q = 0;
    while (q + 1 < g.count && static_cast<int>(blockIdx.x) >= g.prob[q + 1].first_block)
        ++q;
    const GroupRows &r = g.prob[q];
    const int warp = threadIdx.x >> 5;
    const int m = (static_cast<int>(blockIdx.x) - r.first_block) * rows_per_block<WPR>() + warp / WPR;
    // The GEMM that follows may launch at once: a grouped call's grid is
    // small (decode batches), and the GEMM's weight stream needs nothing
    // from this kernel.
    pdl_launch_dependents();
    pdl_wait();
    if (g.clear != nullptr && blockIdx.x == 0)
        for (int i = threadIdx.x; i < g.n_clear; i += THREADS)
            g.clear[i] = 0;
    quant_row<BF16, CACHE, WPR, NORM>(r.x, r.M, r.K, r.xq, r.beta, r.rowsum, r.gain, r.eps, m,
                                      warp % WPR);
}

}  // namespace qa
}  // namespace bitlinear
