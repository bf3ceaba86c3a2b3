// Prefill GEMM: acc = x~ W~^T on the 5th-generation tensor cores
// (tcgen05.mma kind::i8, int32 accumulators in tensor memory).
//
// Pages: "BitNet b1.58 2B4T Guide: Scaling Native 1-Bit LLMs", section
// "Matrix Multiplication as Pure Integer Addition" (the integer contraction
// and the rescale by beta * gamma / 127); "Microsoft Releases BitNet b1.58
// 2B4T", section "The Catch" (GPU kernels must unpack the packed weights).
//
// Tile 128 tokens x 256 weight rows x 128 k per stage; one CTA per SM,
// persistent over tiles (m fastest, so consecutive CTAs share a weight tile
// in L2). Warp roles:
//   warp 0      TMA producer: x~ tile (128 x 128 B, 128-byte swizzle) and the
//               packed weight tile (256 rows x 32 B) into a 4-deep ring;
//   warp 1      MMA issuer (one thread) and TMEM owner (512 columns = two
//               128 x 256 int32 accumulators, so the epilogue of one tile
//               overlaps the MMAs of the next);
//   warps 2-5   epilogue: tcgen05.ld 32 columns at a time, subtract the row
//               sum of x~, rescale by (beta * gamma) / 127, store bf16;
//   warps 6-13  decode: 2-bit codes -> int8 codes {0,1,2} written straight
//               into the 128-byte-swizzled K-major tile the MMA reads.
// The MMA contracts x~ (s8) with the non-negative codes c = W~ + 1 (s8), so
// D = sum x~ c and acc = D - sum_k x~ exactly; no per-byte subtract is needed
// in the decode.
//
// Every mbarrier wait is bounded in time. A wait that runs out records a
// fault word, raises a block-wide abort flag that ends every other wait, and
// each role returns; the producer and the MMA issuer first wait (bounded)
// for their own copies and MMAs in flight, then TMEM is freed.
#pragma once

#include "common.cuh"

namespace bitlinear {
namespace tc {

constexpr int BM = 128;
constexpr int BN = 256;
constexpr int BK = 128;
constexpr int UMMA_K = 32;                 // k per tcgen05.mma kind::i8
constexpr int NS_LOAD = 4;
constexpr int NS_DEC = 3;
constexpr int A_BYTES = BM * BK;           // 16 KiB
constexpr int BP_BYTES = BN * BK / 4;      // 8 KiB
constexpr int BD_BYTES = BN * BK;          // 32 KiB
constexpr int EPI_WARPS = 4;
constexpr int DEC_WARPS = 8;
constexpr int THREADS = (2 + EPI_WARPS + DEC_WARPS) * 32;
constexpr uint32_t TMEM_COLS = 512;
constexpr int NUM_BARS = 2 * NS_LOAD + 2 * NS_DEC + 4 + 2;
constexpr int SMEM_BYTES = 1024 + NS_LOAD * A_BYTES + NS_DEC * BD_BYTES + NS_LOAD * BP_BYTES +
                           NUM_BARS * 8 + 16;
constexpr uint32_t IDESC = idesc_i8_s32(BM, BN);

struct Params {
    int M, N, K;
    float gamma;
    const float *beta;      // [M] (rescale only)
    const int *rowsum;      // [M] sum_k x~ (packed B only)
    uint16_t *y;            // [M][N] bf16 (rescale only)
    int32_t *acc_out;       // [M][N] int32 or null
    uint64_t wait_limit_ns;
    int inject_timeout;     // MMA issuer waits on a barrier nobody arrives at
};

template <bool B_PACKED, bool RESCALE>
__global__ void __launch_bounds__(THREADS, 1)
gemm_kernel(const __grid_constant__ CUtensorMap tmap_a, const __grid_constant__ CUtensorMap tmap_b,
            const Params p)
{
    extern __shared__ uint8_t smem_raw[];
    const uint32_t raw = smem_u32(smem_raw);
    const uint32_t base = (raw + 1023u) & ~1023u;
    uint8_t *const base_ptr = smem_raw + (base - raw);
    const uint32_t sA = base;
    const uint32_t sBd = sA + NS_LOAD * A_BYTES;
    const uint32_t sBp = sBd + NS_DEC * BD_BYTES;
    const uint32_t sBar = sBp + NS_LOAD * BP_BYTES;
    auto bar = [&](int i) -> uint32_t { return sBar + 8u * static_cast<uint32_t>(i); };
    auto full_load = [&](int s) { return bar(s); };
    auto empty_load = [&](int s) { return bar(NS_LOAD + s); };
    auto full_dec = [&](int s) { return bar(2 * NS_LOAD + s); };
    auto empty_dec = [&](int s) { return bar(2 * NS_LOAD + NS_DEC + s); };
    auto tmem_full = [&](int b) { return bar(2 * NS_LOAD + 2 * NS_DEC + b); };
    auto tmem_empty = [&](int b) { return bar(2 * NS_LOAD + 2 * NS_DEC + 2 + b); };
    const uint32_t never_bar = bar(2 * NS_LOAD + 2 * NS_DEC + 4);
    const uint32_t drain_bar = bar(2 * NS_LOAD + 2 * NS_DEC + 5);
    uint32_t *tmem_slot = reinterpret_cast<uint32_t *>(base_ptr + (sBar - base) + NUM_BARS * 8);
    volatile int *abort_flag = reinterpret_cast<volatile int *>(tmem_slot + 1);

    const int warp = threadIdx.x >> 5;
    const int lane = threadIdx.x & 31;
    const uint64_t limit = p.wait_limit_ns;

    if (threadIdx.x == 0) {
        for (int s = 0; s < NS_LOAD; ++s) {
            mbar_init(full_load(s), 1);
            mbar_init(empty_load(s), B_PACKED ? 1 + DEC_WARPS : 1);
        }
        for (int s = 0; s < NS_DEC; ++s) {
            mbar_init(full_dec(s), B_PACKED ? DEC_WARPS : 1);
            mbar_init(empty_dec(s), 1);
        }
        for (int b = 0; b < 2; ++b) {
            mbar_init(tmem_full(b), 1);
            mbar_init(tmem_empty(b), EPI_WARPS);
        }
        mbar_init(never_bar, 1);
        mbar_init(drain_bar, 1);
        *abort_flag = 0;
        fence_barrier_init();
    }
    if (warp == 0 && lane == 0) {
        prefetch_tensormap(&tmap_a);
        prefetch_tensormap(&tmap_b);
    }
    if (warp == 1)
        tmem_alloc(smem_u32(tmem_slot), TMEM_COLS);
    tc_fence_before_sync();
    __syncthreads();
    tc_fence_after_sync();
    const uint32_t tmem_base = *tmem_slot;
    if (warp == 1)
        tmem_relinquish();

    // Tensor-core work may begin only once earlier grids in the stream have
    // finished writing x~ (programmatic dependent launch).
    pdl_wait();

    const int MB = (p.M + BM - 1) / BM;
    const int NB = (p.N + BN - 1) / BN;
    const int KB = p.K / BK;
    const int T = MB * NB;

    if (warp == 0) {
        // ------------------------------------------------------ TMA producer
        if (lane == 0) {
            int ls = 0, ds = 0;
            uint32_t lph = 0, dph = 0;
            int armed_load[NS_LOAD], armed_dec[NS_DEC];
            for (int s = 0; s < NS_LOAD; ++s) armed_load[s] = -1;
            for (int s = 0; s < NS_DEC; ++s) armed_dec[s] = -1;
            for (int t = blockIdx.x; t < T; t += gridDim.x) {
                const int m0 = (t % MB) * BM;
                const int n0 = (t / MB) * BN;
                for (int kb = 0; kb < KB; ++kb) {
                    if (!mbar_wait_bounded(empty_load(ls), lph ^ 1u, abort_flag, limit))
                        goto producer_done;
                    mbar_arrive_expect_tx(full_load(ls), A_BYTES + (B_PACKED ? BP_BYTES : 0));
                    armed_load[ls] = static_cast<int>(lph);
                    tma_load_2d(sA + ls * A_BYTES, &tmap_a, kb * BK, m0, full_load(ls));
                    if constexpr (B_PACKED) {
                        tma_load_4d(sBp + ls * BP_BYTES, &tmap_b, 0, 0, kb, n0 / 16, full_load(ls));
                    } else {
                        if (!mbar_wait_bounded(empty_dec(ds), dph ^ 1u, abort_flag, limit))
                            goto producer_done;
                        mbar_arrive_expect_tx(full_dec(ds), BD_BYTES);
                        armed_dec[ds] = static_cast<int>(dph);
                        tma_load_2d(sBd + ds * BD_BYTES, &tmap_b, kb * BK, n0, full_dec(ds));
                        if (++ds == NS_DEC) { ds = 0; dph ^= 1u; }
                    }
                    if (++ls == NS_LOAD) { ls = 0; lph ^= 1u; }
                }
            }
        producer_done:
            // Wait for every copy this thread started (already complete in a
            // normal run) so no TMA write lands after the block has exited.
            for (int s = 0; s < NS_LOAD; ++s)
                if (armed_load[s] >= 0)
                    drain_wait(full_load(s), static_cast<uint32_t>(armed_load[s]), limit);
            for (int s = 0; s < NS_DEC; ++s)
                if (armed_dec[s] >= 0)
                    drain_wait(full_dec(s), static_cast<uint32_t>(armed_dec[s]), limit);
        }
        __syncwarp();
    } else if (warp == 1) {
        // -------------------------------------------------------- MMA issuer
        if (lane == 0) {
            int ls = 0, ds = 0, lt = 0;
            uint32_t lph = 0, dph = 0;
            if (p.inject_timeout) {
                mbar_wait_bounded(never_bar, 0u, abort_flag, limit);
                goto mma_done;
            }
            for (int t = blockIdx.x; t < T; t += gridDim.x, ++lt) {
                const int buf = lt & 1;
                const uint32_t aph = static_cast<uint32_t>(lt >> 1) & 1u;
                if (!mbar_wait_bounded(tmem_empty(buf), aph ^ 1u, abort_flag, limit))
                    goto mma_done;
                tc_fence_after_sync();
                const uint32_t d_tmem = tmem_base + static_cast<uint32_t>(buf * BN);
                for (int kb = 0; kb < KB; ++kb) {
                    if (!mbar_wait_bounded(full_load(ls), lph, abort_flag, limit))
                        goto mma_done;
                    if (!mbar_wait_bounded(full_dec(ds), dph, abort_flag, limit))
                        goto mma_done;
                    tc_fence_after_sync();
#pragma unroll
                    for (int kk = 0; kk < BK / UMMA_K; ++kk) {
                        const uint64_t adesc = smem_desc_k128_sw128(sA + ls * A_BYTES + kk * UMMA_K);
                        const uint64_t bdesc = smem_desc_k128_sw128(sBd + ds * BD_BYTES + kk * UMMA_K);
                        umma_i8(d_tmem, adesc, bdesc, IDESC, (kb | kk) != 0 ? 1u : 0u);
                    }
                    umma_commit(empty_load(ls));
                    umma_commit(empty_dec(ds));
                    if (++ls == NS_LOAD) { ls = 0; lph ^= 1u; }
                    if (++ds == NS_DEC) { ds = 0; dph ^= 1u; }
                }
                umma_commit(tmem_full(buf));
            }
        mma_done:
            // All MMAs issued by this thread complete before TMEM is freed.
            umma_commit(drain_bar);
            drain_wait(drain_bar, 0u, limit);
        }
        __syncwarp();
    } else if (warp < 2 + EPI_WARPS) {
        // ---------------------------------------------------------- epilogue
        const int q = warp & 3;               // TMEM lane quarter of this warp
        int lt = 0;
        for (int t = blockIdx.x; t < T; t += gridDim.x, ++lt) {
            const int buf = lt & 1;
            const uint32_t aph = static_cast<uint32_t>(lt >> 1) & 1u;
            if (!warp_wait_bounded(tmem_full(buf), aph, abort_flag, limit))
                break;
            tc_fence_after_sync();
            const int m = (t % MB) * BM + q * 32 + lane;
            const int nb0 = (t / MB) * BN;
            float s = 0.0f;
            int rs = 0;
            if (m < p.M) {
                if constexpr (RESCALE) s = out_scale(p.beta[m], p.gamma);
                if constexpr (B_PACKED) rs = p.rowsum[m];
            }
#pragma unroll 1
            for (int c = 0; c < BN / 32; ++c) {
                uint32_t r[32];
                tmem_ld_32x32b_x32(tmem_base + (static_cast<uint32_t>(q * 32) << 16) +
                                       static_cast<uint32_t>(buf * BN + c * 32),
                                   r);
                tmem_ld_wait();
                const int n0 = nb0 + c * 32;
                if (m < p.M && n0 < p.N) {
                    const size_t o = static_cast<size_t>(m) * p.N + n0;
                    const bool full = (n0 + 32 <= p.N);
                    if constexpr (RESCALE) {
                        if (full && (p.N % 8) == 0) {
#pragma unroll
                            for (int g = 0; g < 4; ++g) {
                                uint32_t h[4];
#pragma unroll
                                for (int e = 0; e < 4; ++e) {
                                    const int a0 = static_cast<int>(r[8 * g + 2 * e]) - rs;
                                    const int a1 = static_cast<int>(r[8 * g + 2 * e + 1]) - rs;
                                    h[e] = static_cast<uint32_t>(rescale_bf16(a0, s)) |
                                           (static_cast<uint32_t>(rescale_bf16(a1, s)) << 16);
                                }
                                *reinterpret_cast<uint4 *>(p.y + o + 8 * g) =
                                    make_uint4(h[0], h[1], h[2], h[3]);
                            }
                        } else {
                            for (int e = 0; e < 32 && n0 + e < p.N; ++e)
                                p.y[o + e] = rescale_bf16(static_cast<int>(r[e]) - rs, s);
                        }
                    }
                    if (p.acc_out != nullptr) {
                        if (full && (p.N % 4) == 0) {
#pragma unroll
                            for (int g = 0; g < 8; ++g)
                                *reinterpret_cast<int4 *>(p.acc_out + o + 4 * g) = make_int4(
                                    static_cast<int>(r[4 * g]) - rs, static_cast<int>(r[4 * g + 1]) - rs,
                                    static_cast<int>(r[4 * g + 2]) - rs,
                                    static_cast<int>(r[4 * g + 3]) - rs);
                        } else {
                            for (int e = 0; e < 32 && n0 + e < p.N; ++e)
                                p.acc_out[o + e] = static_cast<int>(r[e]) - rs;
                        }
                    }
                }
            }
            tc_fence_before_sync();
            __syncwarp();
            if (lane == 0)
                mbar_arrive(tmem_empty(buf));
        }
    } else if constexpr (B_PACKED) {
        // ------------------------------------------------------------ decode
        const int dt = (warp - 2 - EPI_WARPS) * 32 + lane;   // 0 .. 255
        int ls = 0, ds = 0;
        uint32_t lph = 0, dph = 0;
        for (int t = blockIdx.x; t < T; t += gridDim.x) {
            for (int kb = 0; kb < KB; ++kb) {
                if (!warp_wait_bounded(full_load(ls), lph, abort_flag, limit))
                    goto decode_done;
                if (!warp_wait_bounded(empty_dec(ds), dph ^ 1u, abort_flag, limit))
                    goto decode_done;
                {
                    const uint32_t *src =
                        reinterpret_cast<const uint32_t *>(base_ptr + (sBp - base) + ls * BP_BYTES);
                    uint8_t *dst = base_ptr + (sBd - base) + ds * BD_BYTES;
#pragma unroll
                    for (int i = 0; i < (BN * BK / 16) / (DEC_WARPS * 32); ++i) {
                        const int widx = dt + i * DEC_WARPS * 32;
                        const int n = widx >> 3;          // 8 words (128 k) per row
                        const int w = widx & 7;
                        const uint32_t word = src[widx];
                        const uint4 o = make_uint4(word & 0x03030303u, (word >> 2) & 0x03030303u,
                                                   (word >> 4) & 0x03030303u,
                                                   (word >> 6) & 0x03030303u);
                        *reinterpret_cast<uint4 *>(dst + (n >> 3) * 1024 + (n & 7) * 128 +
                                                   ((w ^ (n & 7)) << 4)) = o;
                    }
                }
                fence_proxy_async_smem();
                __syncwarp();
                if (lane == 0) {
                    mbar_arrive(full_dec(ds));
                    mbar_arrive(empty_load(ls));
                }
                if (++ls == NS_LOAD) { ls = 0; lph ^= 1u; }
                if (++ds == NS_DEC) { ds = 0; dph ^= 1u; }
            }
        }
    decode_done:;
    }

    // ------------------------------------------------------------ teardown
    tc_fence_before_sync();
    __syncthreads();
    if (warp == 1) {
        tc_fence_after_sync();
        tmem_dealloc(tmem_base, TMEM_COLS);
    }
}

}  // namespace tc
}  // namespace bitlinear
