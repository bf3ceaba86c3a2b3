// Plain int8 GEMM C = A B^T (A [M][K], B [N][K] int8, C [M][N] int32) on the
// 5th-generation tensor cores (tcgen05.mma kind::i8, both operands in shared
// memory, int32 accumulators in tensor memory). It backs bitlinear_int8_gemm,
// a measurement entry point for the integer contraction of page "BitNet
// b1.58 2B4T Guide: Scaling Native 1-Bit LLMs", section "Matrix
// Multiplication as Pure Integer Addition", on already-unpacked operands;
// the BitLinear forward itself uses the weight-stationary GEMM.
//
// Tile 128 x 256 x 128 k per stage; one CTA per SM, persistent over tiles
// (m fastest, so consecutive CTAs share a B tile in L2). Warp roles:
//   warp 0      TMA producer: the A tile (128 x 128 B) and the B tile
//               (256 x 128 B), 128-byte swizzle, into a 4-deep ring;
//   warp 1      MMA issuer (one thread) and TMEM owner (512 columns = two
//               128 x 256 int32 accumulators, so the epilogue of one tile
//               overlaps the MMAs of the next);
//   warps 2-5   epilogue: tcgen05.ld 32 columns at a time, int32 stores.
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
constexpr int NS = 4;
constexpr int A_BYTES = BM * BK;           // 16 KiB
constexpr int B_BYTES = BN * BK;           // 32 KiB
constexpr int EPI_WARPS = 4;
constexpr int THREADS = (2 + EPI_WARPS) * 32;
constexpr uint32_t TMEM_COLS = 512;
constexpr int NUM_BARS = 2 * NS + 4 + 1;
constexpr int SMEM_BYTES = 1024 + NS * (A_BYTES + B_BYTES) + NUM_BARS * 8 + 16;
constexpr uint32_t IDESC = idesc_i8_s32(BM, BN);

struct Params {
    int M, N, K;
    int32_t *c;             // [M][N] int32
    uint64_t wait_limit_ns;
};

__global__ void __launch_bounds__(THREADS, 1)
gemm_kernel(const __grid_constant__ CUtensorMap tmap_a, const __grid_constant__ CUtensorMap tmap_b,
            const Params p)
{
    extern __shared__ uint8_t smem_raw[];
    const uint32_t raw = smem_u32(smem_raw);
    const uint32_t base = (raw + 1023u) & ~1023u;
    uint8_t *const base_ptr = smem_raw + (base - raw);
    const uint32_t sA = base;
    const uint32_t sB = sA + NS * A_BYTES;
    const uint32_t sBar = sB + NS * B_BYTES;
    auto bar = [&](int i) -> uint32_t { return sBar + 8u * static_cast<uint32_t>(i); };
    auto full = [&](int s) { return bar(s); };
    auto empty = [&](int s) { return bar(NS + s); };
    auto tmem_full = [&](int b) { return bar(2 * NS + b); };
    auto tmem_empty = [&](int b) { return bar(2 * NS + 2 + b); };
    const uint32_t drain_bar = bar(2 * NS + 4);
    uint32_t *tmem_slot = reinterpret_cast<uint32_t *>(base_ptr + (sBar - base) + NUM_BARS * 8);
    volatile int *abort_flag = reinterpret_cast<volatile int *>(tmem_slot + 1);

    const int warp = threadIdx.x >> 5;
    const int lane = threadIdx.x & 31;
    const uint64_t limit = p.wait_limit_ns;

    if (threadIdx.x == 0) {
        for (int s = 0; s < NS; ++s) {
            mbar_init(full(s), 1);
            mbar_init(empty(s), 1);
        }
        for (int b = 0; b < 2; ++b) {
            mbar_init(tmem_full(b), 1);
            mbar_init(tmem_empty(b), EPI_WARPS);
        }
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
    pdl_wait();

    const int MB = (p.M + BM - 1) / BM;
    const int NB = (p.N + BN - 1) / BN;
    const int KB = p.K / BK;
    const int T = MB * NB;

    if (warp == 0) {
        // ------------------------------------------------------ TMA producer
        if (lane == 0) {
            int s = 0;
            uint32_t ph = 0;
            int armed[NS];
            for (int i = 0; i < NS; ++i) armed[i] = -1;
            for (int t = blockIdx.x; t < T; t += gridDim.x) {
                const int m0 = (t % MB) * BM;
                const int n0 = (t / MB) * BN;
                for (int kb = 0; kb < KB; ++kb) {
                    if (!mbar_wait_bounded(empty(s), ph ^ 1u, abort_flag, limit))
                        goto producer_done;
                    mbar_arrive_expect_tx(full(s), A_BYTES + B_BYTES);
                    armed[s] = static_cast<int>(ph);
                    tma_load_2d(sA + s * A_BYTES, &tmap_a, kb * BK, m0, full(s));
                    tma_load_2d(sB + s * B_BYTES, &tmap_b, kb * BK, n0, full(s));
                    if (++s == NS) { s = 0; ph ^= 1u; }
                }
            }
        producer_done:
            // Wait for every copy this thread started, so no TMA write lands
            // after the block has exited.
            for (int i = 0; i < NS; ++i)
                if (armed[i] >= 0)
                    drain_wait(full(i), static_cast<uint32_t>(armed[i]), limit);
        }
        __syncwarp();
    } else if (warp == 1) {
        // -------------------------------------------------------- MMA issuer
        if (lane == 0) {
            int s = 0, lt = 0;
            uint32_t ph = 0;
            for (int t = blockIdx.x; t < T; t += gridDim.x, ++lt) {
                const int buf = lt & 1;
                const uint32_t aph = static_cast<uint32_t>(lt >> 1) & 1u;
                if (!mbar_wait_bounded(tmem_empty(buf), aph ^ 1u, abort_flag, limit))
                    goto mma_done;
                tc_fence_after_sync();
                const uint32_t d_tmem = tmem_base + static_cast<uint32_t>(buf * BN);
                for (int kb = 0; kb < KB; ++kb) {
                    if (!mbar_wait_bounded(full(s), ph, abort_flag, limit))
                        goto mma_done;
                    tc_fence_after_sync();
#pragma unroll
                    for (int kk = 0; kk < BK / UMMA_K; ++kk) {
                        const uint64_t adesc = smem_desc_k128_sw128(sA + s * A_BYTES + kk * UMMA_K);
                        const uint64_t bdesc = smem_desc_k128_sw128(sB + s * B_BYTES + kk * UMMA_K);
                        umma_i8(d_tmem, adesc, bdesc, IDESC, (kb | kk) != 0 ? 1u : 0u);
                    }
                    umma_commit(empty(s));
                    if (++s == NS) { s = 0; ph ^= 1u; }
                }
                umma_commit(tmem_full(buf));
            }
        mma_done:
            // All MMAs issued by this thread complete before TMEM is freed.
            umma_commit(drain_bar);
            drain_wait(drain_bar, 0u, limit);
        }
        __syncwarp();
    } else {
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
                    if (n0 + 32 <= p.N && (p.N % 4) == 0) {
#pragma unroll
                        for (int g = 0; g < 8; ++g)
                            *reinterpret_cast<int4 *>(p.c + o + 4 * g) =
                                make_int4(static_cast<int>(r[4 * g]), static_cast<int>(r[4 * g + 1]),
                                          static_cast<int>(r[4 * g + 2]),
                                          static_cast<int>(r[4 * g + 3]));
                    } else {
                        for (int e = 0; e < 32 && n0 + e < p.N; ++e)
                            p.c[o + e] = static_cast<int>(r[e]);
                    }
                }
            }
            tc_fence_before_sync();
            __syncwarp();
            if (lane == 0)
                mbar_arrive(tmem_empty(buf));
        }
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
