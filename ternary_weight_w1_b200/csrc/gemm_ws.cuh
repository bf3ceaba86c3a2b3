// Weight-stationary tensor-core GEMM for the BitLinear forward:
// acc[m][n] = sum_k x~[m][k] * W~[n][k] on tcgen05.mma kind::i8.
//
// Pages: "BitNet b1.58 2B4T Guide: Scaling Native 1-Bit LLMs", section
// "Matrix Multiplication as Pure Integer Addition" (the integer contraction
// and the rescale by beta * gamma / 127); "Microsoft Releases BitNet b1.58
// 2B4T", section "The Catch" (GPU kernels must unpack the packed weights).
//
// The MMA computes D[128 weight rows][BT tokens] = A * B^T with
//   A = decoded weight codes c = W~ + 1 in {0, 1, 2}, held in TENSOR MEMORY:
//       the decode warps unpack the 2-bit codes in registers and write them
//       with tcgen05.st, so decoded weights never pass through shared memory;
//   B = x~ tile [BT tokens][k] in shared memory (TMA, 128-byte swizzle).
// acc = D - sum_k x~[m][k] exactly (the row sums come from the quantiser).
// Because the weights are the MMA's M side, a tile has 128 weight rows and
// BT in {32, 64, 128, 192} tokens, so small token counts still use the
// tensor cores without padding M to 128.
//
// A launch computes one or several independent problems (a problem table of
// up to eight, sharing the token tile); their tiles and k-blocks are numbered
// one problem after the other.
//
// Work split (stream-K): the k-blocks of all tiles are cut into one
// contiguous range per CTA (persistent, one CTA per SM). A tile whose
// k-blocks span two or more CTAs is finished by the CTA holding its first
// k-block: each other CTA stores its int32 partial accumulator [128][BT]
// into its own workspace slot and raises per-warp flags; the finishing CTA
// adds the partials (int32 addition, exact in any order), rescales and
// stores bf16. A CTA stores at most one partial (only the first segment of a
// range can start inside a tile) and finishes tiles only at the end of its
// range, while its contributors write theirs at the start of their ranges.
// Flags are cleared by the quantisation kernel that precedes every GEMM
// launch. Without the split (Params::split = 0) the ranges are whole tiles
// and no partials are used.
//
// A k-block (one pipeline stage) is 256 k, or 512 k for token tiles of 32
// and 64 with enough k-blocks per CTA (deep_stages_fit; the host decides).
// One TMA copy brings the x~ tile of a
// k-block (a 3-D box of 2 or 4 128-byte-swizzled [BT][128] sub-tiles) and
// another the packed weights (a 3-D box of 8 row blocks x 2 or 4 groups x
// 512 bytes). A TMA copy costs the issuing thread about the same time
// whatever its size, so the copies are large and the two streams have a
// producer warp each. A K that is not a multiple of the k-block leaves the
// end of the last k-block outside the tensors, where TMA fills zeros: zero
// x~ and zero codes add nothing.
//
// Warp roles (352 threads; 384 with a second MMA issuer):
//   warp 0     TMA producer of the x~ tiles;
//   warp 1     MMA issuer (one thread) and TMEM owner;
//   warps 2-5  decode: one thread per weight row (TMEM lane), one k-block per stage;
//   warps 6-9  epilogue: tcgen05.ld 32 tokens at a time, partial store or
//              row-sum subtract + rescale to bf16; the [32 tokens][128 rows]
//              bf16 block is transposed through shared memory (two 8 KiB
//              buffers) so that y is written with 16-byte stores;
//   warp 10    TMA producer of the packed weight tiles; it starts before
//              griddepcontrol.wait (no earlier kernel writes the weights);
//   warp 11    second MMA issuer for the 32-token tile (Cfg::DUAL).
// The decode warps wait on a stage's two barriers (copies landed, TMEM slot
// free) at once; the MMA issuer waits only on the decoded-weights barrier,
// since every synchronising wait of that thread idles the tensor pipe.
// TMEM columns: [0, 2 BT) two accumulators (four with two issuers), then the
// NA stages of decoded weights (BK / 4 columns each: four int8 codes per
// column and lane).
//
// Every wait is bounded (mbarriers and inter-CTA flags): on a timeout the
// kernel records a fault word, raises a block-wide abort flag, each role
// returns after draining its own copies and MMAs, and TMEM is freed.
#pragma once

#include "common.cuh"

namespace bitlinear {
namespace wsg {

constexpr int BW = 128;                    // weight rows per tile (MMA M)
constexpr int SUB_K = 128;                 // k per swizzled sub-tile / packed group
constexpr int UMMA_K = 32;                 // k per tcgen05.mma kind::i8

// k per stage (k-block): 256, or 512 for the small token tiles (32 and 64)
// when every CTA has enough k-blocks to fill the deeper stages. A 256-k
// stage of a 32-token tile holds only 364 cycles of MMA (8 MMAs), so there
// a stage's fixed hand-off cost is better paid once per 16 MMAs; the large
// tiles' stages already hold 512 or more cycles and need the shared memory
// for depth, and a launch with few k-blocks per CTA needs its first stage
// early more than it needs fewer stages.
__host__ __device__ constexpr bool deep_stages_fit(int BT) { return BT <= 64; }
constexpr int DEC_WARPS = 4;
constexpr int EPI_WARPS = 4;
constexpr int PK_WARP = 2 + DEC_WARPS + EPI_WARPS;   // second producer
constexpr int MMA2_WARP = PK_WARP + 1;          // second MMA issuer (DUAL launches)
constexpr uint32_t TMEM_COLS = 512;
constexpr int SMEM_BUDGET = 200 * 1024;
constexpr int MAX_GRID = 192;              // upper bound on CTAs (workspace sizing)

template <int BT, int BK_ = 256>
struct Cfg {
    static_assert(BT % 32 == 0 && BT >= 32 && BT <= 224, "token tile");
    // Two MMA-issuing threads (warps 1 and MMA2_WARP) taking alternate
    // stages, each into its own accumulators, for the smallest token tile: a
    // lone issuing thread idles the tensor pipe at every synchronising wait,
    // and short MMAs leave it no time to catch up. At BT = 32 the second pair
    // of accumulators costs no weight stage in TMEM; at BT = 64 it would cost
    // two of six (one of three at BK = 512), which loses more than the
    // second issuer gains.
    static constexpr bool DUAL = BT <= 32;
    static constexpr int ISSUERS = DUAL ? 2 : 1;
    static constexpr int THREADS = (PK_WARP + 1 + (DUAL ? 1 : 0)) * 32;
    static_assert(BK_ == 256 || (BK_ == 512 && deep_stages_fit(BT)), "stage depth");
    static constexpr int BK = BK_;                                 // k per stage
    static constexpr int GROUPS = BK / SUB_K;                      // 128-k groups per stage
    static constexpr int PK_BYTES = BW * BK / 4;                   // packed weights per stage
    static constexpr int A_COLS = BK / 4;                          // TMEM columns per weight stage
    static constexpr int X_SUB = BT * SUB_K;                       // one swizzled sub-tile
    static constexpr int X_BYTES = BT * BK;                        // x~ tile per stage
    static constexpr int STAGE = X_BYTES + PK_BYTES;
    static constexpr int NS = (SMEM_BUDGET / STAGE) < 12 ? (SMEM_BUDGET / STAGE) : 12;
    static constexpr int ACC_COLS = 2 * ISSUERS * BT;              // [issuer][buffer] accumulators
    static constexpr int NA_FIT = (static_cast<int>(TMEM_COLS) - ACC_COLS) / A_COLS;
    static constexpr int NA = NA_FIT < 6 ? NA_FIT : 6;             // TMEM weight stages
    static constexpr int A_COL0 = ACC_COLS;
    static constexpr int NUM_BARS = 2 * NS + 2 * NA + 4 * ISSUERS + 1 + ISSUERS;
    static constexpr int EPI_BYTES = 2 * 32 * BW * 2;              // two bf16 [32][128] blocks
    static constexpr int SMEM_BYTES =
        1024 + NS * X_BYTES + NS * PK_BYTES + EPI_BYTES + NUM_BARS * 8 + 16;
    static constexpr uint32_t IDESC = idesc_i8_s32(BW, BT);
    static_assert(NA >= 2, "TMEM budget");
    static_assert(NS <= 32, "slot masks");
    static_assert(SMEM_BYTES <= 227 * 1024, "shared memory budget");
};

constexpr int MAX_PROBLEMS = 8;

// One matmul of a launch. A launch runs one or several independent problems
// (sharing the token tile BT); their tiles and k-blocks are numbered one
// after the other.
struct Problem {
    int M, N;               // tokens, weight rows
    int MT, KB;             // token tiles; k-blocks (256 k) per tile: ceil(K / 256)
    int iter_begin;         // global index of the problem's first k-block
    int tile_begin;         // global index of the problem's first tile
    float gamma;
    const float *beta;      // [M]
    const int *rowsum;      // [M] sum_k x~
    uint16_t *y;            // [M][N] bf16
    int32_t *acc_out;       // [M][N] int32 or null
};

// TMA descriptors of every problem's x~ and packed weights.
struct Maps {
    CUtensorMap x[MAX_PROBLEMS];
    CUtensorMap w[MAX_PROBLEMS];
};

struct Params {
    Problem prob[MAX_PROBLEMS];
    int count;
    int total_iters, total_tiles;
    int32_t *partial;       // [grid][BW][BT] int32 (split only)
    int *flags;             // [grid][4] zero at launch (split only)
    int split;              // 1: CTA ranges in k-blocks (stream-K); 0: in whole tiles
    int base, extra;        // units per CTA: base, plus one for the first `extra`
    uint64_t wait_limit_ns;
    int inject_timeout;     // MMA issuer waits on a barrier nobody arrives at
};

// The problem holding global k-block `it` / global tile `tile`.
__device__ __forceinline__ int problem_of_iter(const Params &p, int it)
{
    int q = 0;
    while (q + 1 < p.count && it >= p.prob[q + 1].iter_begin)
        ++q;
    return q;
}

__device__ __forceinline__ int problem_of_tile(const Params &p, int tile)
{
    int q = 0;
    while (q + 1 < p.count && tile >= p.prob[q + 1].tile_begin)
        ++q;
    return q;
}

// First global k-block of CTA c's range.
__device__ __forceinline__ int range_begin(const Params &p, int c)
{
    const int u = c * p.base + min(c, p.extra);
    if (p.split)
        return u;
    if (u >= p.total_tiles)
        return p.total_iters;
    const int q = problem_of_tile(p, u);
    return p.prob[q].iter_begin + (u - p.prob[q].tile_begin) * p.prob[q].KB;
}

// The CTA whose range holds global k-block `it` (stream-K ranges only).
__device__ __forceinline__ int range_owner(const Params &p, int it)
{
    const int big = p.extra * (p.base + 1);
    return it < big ? it / (p.base + 1) : p.extra + (it - big) / p.base;
}

template <int BT, int BK = 256>
__global__ void __launch_bounds__((Cfg<BT, BK>::THREADS), 1)
gemm_ws_kernel(const __grid_constant__ Maps maps, const __grid_constant__ Params p)
{
    using C = Cfg<BT, BK>;
    constexpr int NS = C::NS;
    constexpr int NA = C::NA;
    extern __shared__ uint8_t smem_raw[];
    const uint32_t raw = smem_u32(smem_raw);
    const uint32_t base = (raw + 1023u) & ~1023u;
    uint8_t *const base_ptr = smem_raw + (base - raw);
    const uint32_t sX = base;
    const uint32_t sP = sX + NS * C::X_BYTES;
    constexpr int PK_BYTES = C::PK_BYTES;
    const uint32_t sEpi = sP + NS * PK_BYTES;
    const uint32_t sBar = sEpi + C::EPI_BYTES;
    auto bar = [&](int i) -> uint32_t { return sBar + 8u * static_cast<uint32_t>(i); };
    auto full_load = [&](int s) { return bar(s); };
    auto empty_load = [&](int s) { return bar(NS + s); };
    auto a_full = [&](int a) { return bar(2 * NS + a); };
    auto a_empty = [&](int a) { return bar(2 * NS + NA + a); };
    constexpr int ISSUERS = C::ISSUERS;
    // accumulator barriers per issuer i and buffer b
    auto acc_full = [&](int i, int b) { return bar(2 * NS + 2 * NA + 2 * i + b); };
    auto acc_empty = [&](int i, int b) { return bar(2 * NS + 2 * NA + 2 * ISSUERS + 2 * i + b); };
    const uint32_t never_bar = bar(2 * NS + 2 * NA + 4 * ISSUERS);
    auto drain_bar = [&](int i) { return bar(2 * NS + 2 * NA + 4 * ISSUERS + 1 + i); };
    uint32_t *tmem_slot = reinterpret_cast<uint32_t *>(base_ptr + (sBar - base) + C::NUM_BARS * 8);
    volatile int *abort_flag = reinterpret_cast<volatile int *>(tmem_slot + 1);

    const int warp = threadIdx.x >> 5;
    const int lane = threadIdx.x & 31;
    const uint64_t limit = p.wait_limit_ns;

    if (threadIdx.x == 0) {
        for (int s = 0; s < NS; ++s) {
            mbar_init(full_load(s), 2);
            mbar_init(empty_load(s), 1 + DEC_WARPS);
        }
        for (int a = 0; a < NA; ++a) {
            mbar_init(a_full(a), DEC_WARPS);
            mbar_init(a_empty(a), 1);
        }
        for (int i = 0; i < ISSUERS; ++i) {
            for (int b = 0; b < 2; ++b) {
                mbar_init(acc_full(i, b), 1);
                mbar_init(acc_empty(i, b), EPI_WARPS);
            }
            mbar_init(drain_bar(i), 1);
        }
        mbar_init(never_bar, 1);
        *abort_flag = 0;
        fence_barrier_init();
    }
    if (warp == 0 && lane < p.count)
        prefetch_tensormap(&maps.x[lane]);
    if (warp == PK_WARP && lane < p.count)
        prefetch_tensormap(&maps.w[lane]);
    if (warp == 1)
        tmem_alloc(smem_u32(tmem_slot), TMEM_COLS);
    tc_fence_before_sync();
    __syncthreads();
    tc_fence_after_sync();
    const uint32_t tmem_base = *tmem_slot;
    if (warp == 1)
        tmem_relinquish();

    // x~, beta, the row sums and the flags are written by the preceding
    // quantisation kernel (programmatic dependent launch). The packed
    // weights are not: their producer starts streaming at once.
    if (warp != PK_WARP)
        pdl_wait();

    const int it_begin = range_begin(p, blockIdx.x);
    const int it_end = range_begin(p, blockIdx.x + 1);

    if (warp == 0 || warp == PK_WARP) {
        // ----------------------------------------------------- TMA producers
        // warp 0 copies the x~ tiles, warp PK_WARP the packed weight tiles;
        // each arms the stage's full barrier with its own byte count.
        if (lane == 0) {
            const bool is_x = (warp == 0);
            int s = 0;
            uint32_t ph = 0;
            uint32_t armed = 0, armed_ph = 0;   // slots armed (bit i) and their phase
            // The stage's coordinates are stepped, not recomputed: problem q,
            // its k-block kb and tile t = nt * MT + mt (the token tile varies
            // fastest). A lone thread issues the copies, and the loop's own
            // latency (parameter reads, divisions) would otherwise pace it.
            int q = problem_of_iter(p, it_begin);
            int kb = 0, mt = 0, nt = 0, KB = 1, MT = 1;
            const CUtensorMap *map = nullptr;
            auto enter = [&](int it) {
                const Problem &P = p.prob[q];
                KB = P.KB;
                MT = P.MT;
                const int local = it - P.iter_begin;
                const int t = local / KB;
                kb = local - t * KB;
                mt = t % MT;
                nt = t / MT;
                map = is_x ? &maps.x[q] : &maps.w[q];
            };
            if (it_begin < it_end)
                enter(it_begin);
            int next_begin = q + 1 < p.count ? p.prob[q + 1].iter_begin : it_end;
            for (int it = it_begin; it < it_end; ++it) {
                if (it >= next_begin) {
                    // first k-block of a later problem (skipping empty ones)
                    do {
                        ++q;
                    } while (q + 1 < p.count && it >= p.prob[q + 1].iter_begin);
                    enter(it);
                    next_begin = q + 1 < p.count ? p.prob[q + 1].iter_begin : it_end;
                }
                if (!mbar_wait_bounded(empty_load(s), ph ^ 1u, abort_flag, limit))
                    break;
                armed |= 1u << s;
                armed_ph = (armed_ph & ~(1u << s)) | (ph << s);
                if (is_x) {
                    mbar_arrive_expect_tx(full_load(s), C::X_BYTES);
                    tma_load_3d(sX + s * C::X_BYTES, map, 0, mt * BT, C::GROUPS * kb,
                                full_load(s));
                } else {
                    mbar_arrive_expect_tx(full_load(s), PK_BYTES);
                    tma_load_3d(sP + s * PK_BYTES, map, 0, C::GROUPS * kb, nt * (BW / 16),
                                full_load(s));
                }
                if (++kb == KB) {
                    kb = 0;
                    if (++mt == MT) { mt = 0; ++nt; }
                }
                if (++s == NS) { s = 0; ph ^= 1u; }
            }
            // Wait for every copy this thread started, so no TMA write lands
            // after the block has exited.
            for (int i = 0; i < NS; ++i)
                if (armed & (1u << i))
                    drain_wait(full_load(i), (armed_ph >> i) & 1u, limit);
        }
        __syncwarp();
    } else if (warp == 1 || (C::DUAL && warp == MMA2_WARP)) {
        // -------------------------------------------------------- MMA issuer
        // Issuer me takes this CTA's stages c with c % ISSUERS == me, into
        // its own accumulator pair; the epilogue adds the issuers' sums.
        if (lane == 0) {
            const int me = (warp == 1) ? 0 : 1;
            int seg = 0;
            // The x~ descriptors of every stage and k-step differ from stage
            // 0's first one only in the start address (low word, 16-byte
            // units, no carry: shared addresses stay below 2^18), so the
            // issuing loop adds constants instead of rebuilding 64-bit
            // descriptors: a lone thread has no other work to hide the
            // latency of that arithmetic behind.
            const uint64_t bdesc0 = smem_desc_k128_sw128(sX);
            const uint32_t b_lo0 = static_cast<uint32_t>(bdesc0);
            const uint32_t b_hi = static_cast<uint32_t>(bdesc0 >> 32);
            if (p.inject_timeout) {
                mbar_wait_bounded(never_bar, 0u, abort_flag, limit);
                goto mma_done;
            }
            for (int it = it_begin; it < it_end; ++seg) {
                const Problem &P = p.prob[problem_of_iter(p, it)];
                const int local = it - P.iter_begin;
                const int t = local / P.KB;
                const int k0 = local - t * P.KB;
                const int k1 = min(P.KB, k0 + (it_end - it));
                const int buf = seg & 1;
                if (!mbar_wait_bounded(acc_empty(me, buf),
                                       ((static_cast<uint32_t>(seg) >> 1) & 1u) ^ 1u, abort_flag,
                                       limit))
                    goto mma_done;
                tc_fence_after_sync();
                const uint32_t d_tmem =
                    tmem_base + static_cast<uint32_t>((2 * me + buf) * BT);
                bool first = true;
                for (int kb = k0; kb < k1; ++kb) {
                    const int c = it - it_begin + (kb - k0);   // this CTA's stage number
                    if (ISSUERS > 1 && (c % ISSUERS) != me)
                        continue;
                    const int s = c % NS;
                    const int a = c % NA;
                    const uint32_t aph = static_cast<uint32_t>(c / NA) & 1u;
                    // a_full(a) completes only after the decode warps have
                    // seen full_load(s) (both TMA copies of the stage, x~
                    // included, have landed) and written the codes, so one
                    // wait covers both operands. Waiting on the transaction
                    // barrier here as well costs the issuing thread more than
                    // the short MMA queue holds.
                    if (!mbar_wait_bounded(a_full(a), aph, abort_flag, limit))
                        goto mma_done;
                    tc_fence_after_sync();
                    const uint32_t a_tmem =
                        tmem_base + static_cast<uint32_t>(C::A_COL0 + C::A_COLS * a);
                    const uint32_t b_lo = b_lo0 + static_cast<uint32_t>(s * (C::X_BYTES >> 4));
                    const uint32_t acc_in = first ? 0u : 1u;
#pragma unroll
                    for (int kk = 0; kk < C::BK / UMMA_K; ++kk) {
                        constexpr int X_SUB16 = C::X_SUB >> 4;
                        umma_i8_tmem_a_w(d_tmem, a_tmem + static_cast<uint32_t>(8 * kk),
                                         b_lo + static_cast<uint32_t>((kk / 4) * X_SUB16 +
                                                                      (kk % 4) * (UMMA_K >> 4)),
                                         b_hi, C::IDESC, kk > 0 ? 1u : acc_in);
                    }
                    first = false;
                    umma_commit(empty_load(s));
                    umma_commit(a_empty(a));
                }
                // arrives once this issuer's MMAs of the segment are done (at
                // once when it had none: the epilogue then skips its sum)
                umma_commit(acc_full(me, buf));
                it += k1 - k0;
            }
        mma_done:
            // All MMAs issued by this thread complete before TMEM is freed.
            umma_commit(drain_bar(me));
            drain_wait(drain_bar(me), 0u, limit);
        }
        __syncwarp();
    } else if (warp < 2 + DEC_WARPS) {
        // ------------------------------------------------------------ decode
        // Thread = weight row r of the tile = TMEM lane r. The packed stage
        // is [8 row blocks][2 groups][16 rows][32 B]; in group g, word w of
        // row r has k = 128 g + 16 w + 4 j + b at bits 8 b + 2 j, so plane j
        // of word w goes to TMEM column 32 g + 4 w + j (four k per column,
        // k = 4 c + b in byte b).
        const int q = warp & 3;
        const int r = 32 * q + lane;
        const uint32_t lane_off = static_cast<uint32_t>(32 * q) << 16;
        const int row_off = (r >> 4) * (C::GROUPS * 512) + (r & 15) * 32;
        int s = 0, a = 0;
        uint32_t ph = 0, aph = 0;
        for (int it = it_begin; it < it_end; ++it) {
            // the stage's copies have landed and its TMEM slot is free
            if (!warp_wait2_bounded(full_load(s), ph, a_empty(a), aph ^ 1u, abort_flag, limit))
                break;
            tc_fence_after_sync();
            const uint8_t *stage = base_ptr + (sP - base) + s * PK_BYTES + row_off;
            // All of the stage's packed words are loaded before the first
            // TMEM store: the stores are asm statements the compiler does not
            // move loads across, so loads interleaved with them would wait out
            // one shared-memory latency per group.
            uint4 wv[2 * C::GROUPS];
#pragma unroll
            for (int g = 0; g < C::GROUPS; ++g) {
                wv[2 * g] = *reinterpret_cast<const uint4 *>(stage + 512 * g);
                wv[2 * g + 1] = *reinterpret_cast<const uint4 *>(stage + 512 * g + 16);
            }
#pragma unroll
            for (int g = 0; g < C::GROUPS; ++g) {
                const uint4 w0 = wv[2 * g];
                const uint4 w1 = wv[2 * g + 1];
                const uint32_t wd[8] = {w0.x, w0.y, w0.z, w0.w, w1.x, w1.y, w1.z, w1.w};
                uint32_t v[32];
#pragma unroll
                for (int w = 0; w < 8; ++w) {
                    v[4 * w + 0] = wd[w] & 0x03030303u;
                    v[4 * w + 1] = (wd[w] >> 2) & 0x03030303u;
                    v[4 * w + 2] = (wd[w] >> 4) & 0x03030303u;
                    v[4 * w + 3] = (wd[w] >> 6) & 0x03030303u;
                }
                tmem_st_32x32b_x32(
                    tmem_base + lane_off +
                        static_cast<uint32_t>(C::A_COL0 + C::A_COLS * a + 32 * g), v);
            }
            tmem_st_wait();
            tc_fence_before_sync();
            __syncwarp();
            if (lane == 0) {
                mbar_arrive(a_full(a));
                mbar_arrive(empty_load(s));
            }
            if (++s == NS) { s = 0; ph ^= 1u; }
            if (++a == NA) { a = 0; aph ^= 1u; }
        }
    } else {
        // ---------------------------------------------------------- epilogue
        const int q = warp & 3;
        const int row = 32 * q + lane;                      // weight row in the tile
        const uint32_t lane_off = static_cast<uint32_t>(32 * q) << 16;
        int seg = 0;
        int epi_chunk = 0;                 // alternates the two transpose buffers
        for (int it = it_begin; it < it_end; ++seg) {
            const Problem &P = p.prob[problem_of_iter(p, it)];
            const int local = it - P.iter_begin;
            const int t = local / P.KB;
            const int k0 = local - t * P.KB;
            const int k1 = min(P.KB, k0 + (it_end - it));
            // which issuers have stages in this segment (with two, a segment
            // of one stage belongs to the issuer of its parity)
            const int c0 = it - it_begin;
            const bool has0 = ISSUERS == 1 || k1 - k0 >= 2 || (c0 & 1) == 0;
            const bool has1 = ISSUERS == 2 && (k1 - k0 >= 2 || (c0 & 1) == 1);
            it += k1 - k0;
            const int buf = seg & 1;
            const int mt = t % P.MT;
            const int nt = t / P.MT;

            // Per-token scale and row sum of this tile, fetched before the
            // accumulator is ready: lane l holds token mt * BT + 32 c + l.
            float s_pf[BT / 32];
            int rs_pf[BT / 32];
            if (k0 == 0) {
#pragma unroll
                for (int c = 0; c < BT / 32; ++c) {
                    const int ml = mt * BT + 32 * c + lane;
                    s_pf[c] = ml < P.M ? out_scale(__ldg(P.beta + ml), P.gamma) : 0.0f;
                    rs_pf[c] = ml < P.M ? __ldg(P.rowsum + ml) : 0;
                }
            }

            // The four epilogue warps take every wait's verdict together (named
            // barrier 1), so none can be left behind at the transpose barrier.
            const uint32_t acc_par = (static_cast<uint32_t>(seg) >> 1) & 1u;
            bool ready = ISSUERS == 1
                             ? warp_wait_bounded(acc_full(0, buf), acc_par, abort_flag, limit)
                             : warp_wait2_bounded(acc_full(0, buf), acc_par,
                                                  acc_full(ISSUERS - 1, buf), acc_par, abort_flag,
                                                  limit);
            if (!named_bar_and(1, EPI_WARPS * 32, ready))
                break;
            tc_fence_after_sync();
            // chunk c of the segment's sum: issuer 0's accumulator plus, with
            // two issuers, issuer 1's (only the issuers that had stages)
            auto load_acc = [&](int c, uint32_t (&r)[32]) {
                const uint32_t col = lane_off + static_cast<uint32_t>(32 * c);
                if (has0)
                    tmem_ld_32x32b_x32(tmem_base + col + static_cast<uint32_t>(buf * BT), r);
                if constexpr (ISSUERS == 2) {
                    if (has1) {
                        uint32_t r1[32];
                        tmem_ld_32x32b_x32(
                            tmem_base + col + static_cast<uint32_t>((2 + buf) * BT), r1);
                        tmem_ld_wait();
#pragma unroll
                        for (int j = 0; j < 32; ++j)
                            r[j] = has0 ? r[j] + r1[j] : r1[j];
                    }
                }
                tmem_ld_wait();
            };
            auto release_acc = [&]() {
                if (lane == 0)
                    for (int i = 0; i < ISSUERS; ++i)
                        mbar_arrive(acc_empty(i, buf));
            };

            if (k0 > 0) {
                // Not the tile's first k-block: hand the partial sum to the
                // CTA that finishes the tile.
                int32_t *slot = p.partial + (static_cast<size_t>(blockIdx.x) * BW + row) * BT;
#pragma unroll 1
                for (int c = 0; c < BT / 32; ++c) {
                    uint32_t r[32];
                    load_acc(c, r);
#pragma unroll
                    for (int g = 0; g < 8; ++g)
                        __stcg(reinterpret_cast<int4 *>(slot + 32 * c + 4 * g),
                               make_int4(static_cast<int>(r[4 * g]), static_cast<int>(r[4 * g + 1]),
                                         static_cast<int>(r[4 * g + 2]),
                                         static_cast<int>(r[4 * g + 3])));
                }
                // The warp barrier orders every lane's stores before lane 0's
                // release of the flag (a release is cumulative).
                tc_fence_before_sync();
                __syncwarp();
                if (lane == 0)
                    st_release_gpu(p.flags + 4 * blockIdx.x + q, 1);
                release_acc();
                continue;
            }

            // First k-block of the tile is here: this CTA finishes the tile.
            // Other contributors: the CTAs holding the tile's later k-blocks.
            const int c_last = (k1 < P.KB) ? range_owner(p, P.iter_begin + (t + 1) * P.KB - 1)
                                           : static_cast<int>(blockIdx.x);
            // Every lane polls some of the contributors' flags (lane l takes
            // contributors blockIdx.x + 1 + l, + 33, ...), so all of them are
            // read in one round trip when they are already set.
            bool ok = true;
            const int n_contrib = c_last - static_cast<int>(blockIdx.x);
            if (n_contrib > 0) {
                const uint64_t t0 = global_timer_ns();
                for (uint32_t spin = 0;; ++spin) {
                    bool mine = true;
                    for (int c2 = blockIdx.x + 1 + lane; c2 <= c_last; c2 += 32)
                        mine = mine && (ld_acquire_gpu(p.flags + 4 * c2 + q) != 0);
                    if (__all_sync(0xffffffffu, mine))
                        break;
                    if ((spin & 15u) == 15u) {
                        int stop = 0;
                        if (lane == 0) {
                            if (*abort_flag) {
                                stop = 1;
                            } else if (global_timer_ns() - t0 > limit) {
                                atomicOr(&g_fault_word, FAULT_WAIT_TIMEOUT);
                                *abort_flag = 1;
                                stop = 1;
                            }
                        }
                        if (__shfl_sync(0xffffffffu, stop, 0)) {
                            ok = false;
                            break;
                        }
                    }
                }
                // Each flag was read with acquire semantics by some lane; the
                // warp barrier orders those reads before every lane's loads.
                __syncwarp();
            }
            if (!named_bar_and(1, EPI_WARPS * 32, ok))
                break;

            const int n = nt * BW + row;
            const bool n_ok = n < P.N;
            const bool vec_out = (P.N % 8) == 0;
#pragma unroll
            for (int c = 0; c < BT / 32; ++c) {
                const int m0 = mt * BT + 32 * c;
                if (m0 >= P.M)
                    break;
                uint32_t r[32];
                load_acc(c, r);
                // Partial sums of the other contributors, two at a time so
                // that their loads are in flight together.
                for (int c2 = blockIdx.x + 1; c2 <= c_last; c2 += 2) {
                    const bool two = (c2 + 1 <= c_last);
                    const int4 *sa = reinterpret_cast<const int4 *>(
                        p.partial + (static_cast<size_t>(c2) * BW + row) * BT + 32 * c);
                    const int4 *sb = reinterpret_cast<const int4 *>(
                        p.partial + (static_cast<size_t>(two ? c2 + 1 : c2) * BW + row) * BT + 32 * c);
                    int4 va[8], vb[8];
#pragma unroll
                    for (int g = 0; g < 8; ++g) {
                        va[g] = __ldcg(sa + g);
                        vb[g] = two ? __ldcg(sb + g) : make_int4(0, 0, 0, 0);
                    }
#pragma unroll
                    for (int g = 0; g < 8; ++g) {
                        r[4 * g] += static_cast<uint32_t>(va[g].x + vb[g].x);
                        r[4 * g + 1] += static_cast<uint32_t>(va[g].y + vb[g].y);
                        r[4 * g + 2] += static_cast<uint32_t>(va[g].z + vb[g].z);
                        r[4 * g + 3] += static_cast<uint32_t>(va[g].w + vb[g].w);
                    }
                }
                const int jn = min(32, P.M - m0);
                if (P.acc_out != nullptr) {
#pragma unroll
                    for (int j = 0; j < 32; ++j) {
                        const int rs = __shfl_sync(0xffffffffu, rs_pf[c], j);
                        if (j < jn && n_ok)
                            P.acc_out[static_cast<size_t>(m0 + j) * P.N + n] =
                                static_cast<int>(r[j]) - rs;
                    }
                }
                if (vec_out) {
                    // [32 tokens][128 rows] bf16 block in shared memory, then
                    // 16-byte stores: 16 lanes cover one token's 256 bytes.
                    uint16_t *blk = reinterpret_cast<uint16_t *>(
                        base_ptr + (sEpi - base) + (epi_chunk & 1) * (32 * BW * 2));
#pragma unroll
                    for (int j = 0; j < 32; ++j) {
                        const float s = __shfl_sync(0xffffffffu, s_pf[c], j);
                        const int rs = __shfl_sync(0xffffffffu, rs_pf[c], j);
                        blk[j * BW + row] = rescale_bf16(static_cast<int>(r[j]) - rs, s);
                    }
                    asm volatile("bar.sync 1, %0;" ::"r"(EPI_WARPS * 32) : "memory");
                    const int et = (warp - 2 - DEC_WARPS) * 32 + lane;   // 0 .. 127
#pragma unroll
                    for (int i = 0; i < 4; ++i) {
                        const int sg = et + 128 * i;                    // 16-byte segment
                        const int j = sg >> 4;
                        const int piece = sg & 15;
                        const int nn = nt * BW + 8 * piece;
                        if (j < jn && nn < P.N) {
                            const uint4 v = *reinterpret_cast<const uint4 *>(blk + j * BW + 8 * piece);
                            *reinterpret_cast<uint4 *>(P.y + static_cast<size_t>(m0 + j) * P.N + nn) = v;
                        }
                    }
                    ++epi_chunk;
                } else {
                    uint16_t *yrow = P.y + static_cast<size_t>(m0) * P.N + n;
#pragma unroll
                    for (int j = 0; j < 32; ++j) {
                        const float s = __shfl_sync(0xffffffffu, s_pf[c], j);
                        const int rs = __shfl_sync(0xffffffffu, rs_pf[c], j);
                        if (j < jn && n_ok)
                            yrow[static_cast<size_t>(j) * P.N] =
                                rescale_bf16(static_cast<int>(r[j]) - rs, s);
                    }
                }
            }
            tc_fence_before_sync();
            __syncwarp();
            release_acc();
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

}  // namespace wsg
}  // namespace bitlinear
