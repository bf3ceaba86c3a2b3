// Decode GEMV for small M: y = BitLinear(x) with the activation quantisation
// fused in the prologue and the packed ternary weights streamed from HBM once.
//
// Pages: "BitNet b1.58 2B4T Guide: Scaling Native 1-Bit LLMs", sections
// "8-Bit Activation Quantization: absmax Scaling" (prologue), "Matrix
// Multiplication as Pure Integer Addition" (contraction and rescale); the
// memory-wall framing of "BitNet b1.58: The 1-Bit Paradigm Shift" is why the
// kernel is organised around the weight bytes.
//
// Work split. The packed layout keeps 16-row blocks contiguous, so block b of
// the grid owns q whole row blocks = one contiguous byte range. A producer
// warp streams that range through a ring of 8 KiB shared-memory slots with
// bulk (TMA) copies, starting before the programmatic-launch wait so the weight
// stream overlaps the previous kernel and this kernel's prologue. Eight
// compute warps consume 512-byte pieces (one row block x one k-group of 128
// weights: 16 rows x 32 B) round-robin; lane (r, t) = (lane / 2, lane % 2)
// always holds row r of the piece and the k-half t, i.e. 64 weights, so the
// activations it needs are one 64-byte run of x~ that all 16 rows share (a
// two-address broadcast read from shared memory).
//
// Arithmetic. With codes c = W~ + 1 in {0,1,2}, the four 2-bit fields j of
// each byte of a packed word w hold the weights k = 16w' + 4j .. 16w' + 4j + 3
// of its 16-weight run. w & 0x03030303 and w & 0x0C0C0C0C leave c and 4c in
// every byte for j = 0 and 1, and the same two masks on w >> 4 do it for
// j = 2 and 3: all values fit a signed byte, so one signed dp4a per 4 weights
// and token multiplies them with the matching x~ word. The two accumulators
// (scale 1: j = 0, 2; scale 4: j = 1, 3) give
//   sum c*x~ = s1 + (s4 >> 2)
// exactly (s4 is a multiple of 4), and acc = sum c*x~ - sum x~ (the token's
// sum of x~ comes from the prologue). Each piece's partial is folded with the
// k-half partner lane by one shuffle and added into a per-row int32
// shared-memory accumulator (integer, so the order of the atomic adds cannot
// change the result); pieces are therefore independent, and each warp works
// on all of its pieces of a ring slot at once, without branches.
//
// RMS normalisation (NORM launches). The listing's BitLinear normalises each
// token with its nn.RMSNorm member before quantising it; here that is one more
// prologue pass. Each thread sums the squares of its activations in double
// (exact products), the warps' sums go to shared memory and every thread adds
// them in the same order, so all CTAs derive the same r = 1 / sqrt(mean +
// eps); the absmax and quantisation passes then work on (x * r) * g.
//
// Every mbarrier wait is bounded; a wait that runs out records the fault word
// and lets every warp return (the producer first waits for its own copies).
#pragma once

#include "common.cuh"

namespace bitlinear {
namespace gemv {

constexpr int CWARPS = 8;                          // compute warps
constexpr int CTHREADS = CWARPS * 32;
constexpr int THREADS = CTHREADS + 32;             // + the producer warp
constexpr int PIECE = 512;                         // one (row block, k-group)
constexpr int STAGE = 16384;                       // bytes per ring slot
constexpr int PIECES_PER_STAGE = STAGE / PIECE;
constexpr int PIECES_PER_WARP = PIECES_PER_STAGE / CWARPS;   // per stage
constexpr int MAX_SLOTS = 16;
constexpr int BAR_BYTES = 2 * MAX_SLOTS * 8 + 16;  // full/empty barriers + abort flag

constexpr int MAX_PROBLEMS = 8;

// One BitLinear problem of a GEMV launch; a launch may carry several
// independent problems (a grouped launch), each with its own CTAs.
struct Problem {
    const void *x;
    const uint8_t *packed;
    uint16_t *y;
    int32_t *acc_dbg;
    int8_t *xq_dbg;
    float *beta_dbg;
    int M, K, N;
    float gamma;
    const float *norm_gain; // [K] RMS-normalisation gains (NORM launches only)
    float norm_eps;         // eps of the normalisation (NORM launches only)
    int blocks_per_cta;     // row blocks of 16 rows owned by one CTA
    int cta_begin;          // this problem's first CTA in the grid
    uint64_t kg_magic;      // ceil(2^32 / (K / 128)): i / KG == (i * kg_magic) >> 32
                            // for every piece index i < 2^23 at any KG <= 512 (the
                            // host keeps blocks_per_cta * KG below that)
};

struct Params {
    Problem prob[MAX_PROBLEMS];
    int count;              // problems in this launch
    int slots;              // ring slots (<= MAX_SLOTS)
    int xq_cap;             // shared bytes for x~: max over problems of M * K
    int acc_cap;            // row accumulators: max over problems of blocks_per_cta * 16 * MT
    uint64_t wait_limit_ns;
};

__host__ __device__ constexpr int smem_bytes(int MT, int xq_cap, int acc_cap, int slots,
                                             bool norm = false)
{
    return slots * STAGE + BAR_BYTES + xq_cap + acc_cap * 4 + (norm ? MT * CWARPS * 8 : 0) +
           MT * 4 + 2 * MT * CWARPS * 4;
}

// r of token m from the warps' partial sums of squares, added in warp order.
__device__ __forceinline__ float row_rms_scale(const double *red_d, int m, int K, float eps)
{
    double ss = red_d[m * CWARPS];
#pragma unroll
    for (int w = 1; w < CWARPS; ++w)
        ss = __dadd_rn(ss, red_d[m * CWARPS + w]);
    return rms_scale(ss, K, eps);
}

__device__ __forceinline__ void compute_sync()
{
    asm volatile("bar.sync 1, %0;" ::"r"(CTHREADS) : "memory");
}

// Three blocks per SM fit the register file (two of this grid and, under
// programmatic dependent launch, one of the next).
template <int MT, bool BF16, bool NORM>
__global__ void __launch_bounds__(THREADS, 3)
gemv_kernel(const __grid_constant__ Params p)
{
    extern __shared__ __align__(128) uint8_t smem[];
    // this CTA's problem (grouped launches give each problem its own CTAs)
    int pi = 0;
#pragma unroll 1
    while (pi + 1 < p.count && static_cast<int>(blockIdx.x) >= p.prob[pi + 1].cta_begin)
        ++pi;
    const Problem &P = p.prob[pi];
    const int K = P.K, M = P.M, N = P.N;
    const int KG = K >> 7;                              // k-groups per row
    const int total_blocks = (N + 15) >> 4;
    const int q = P.blocks_per_cta;
    const int blk0 = (static_cast<int>(blockIdx.x) - P.cta_begin) * q;
    const int nblk = min(q, total_blocks - blk0);
    const size_t block_bytes = static_cast<size_t>(K) * 4;   // 16 rows x K/4 bytes
    const uint8_t *src = P.packed + static_cast<size_t>(blk0) * block_bytes;
    const int npieces = nblk * KG;
    const int nstages = (npieces + PIECES_PER_STAGE - 1) / PIECES_PER_STAGE;
    const int slots = p.slots;

    uint8_t *ring = smem;
    const uint32_t bars = smem_u32(smem + slots * STAGE);
    auto full = [&](int s) { return bars + 8u * static_cast<uint32_t>(s); };
    auto empty = [&](int s) { return bars + 8u * static_cast<uint32_t>(MAX_SLOTS + s); };
    volatile int *abort_flag =
        reinterpret_cast<volatile int *>(smem + slots * STAGE + 2 * MAX_SLOTS * 8);
    uint8_t *xq_sm = smem + slots * STAGE + BAR_BYTES;
    int *acc_sm = reinterpret_cast<int *>(xq_sm + p.xq_cap);
    // [MT][CWARPS] partial sums of squares (NORM only; 8-byte aligned: every
    // region before it is a multiple of 8 bytes)
    double *red_d = reinterpret_cast<double *>(acc_sm + p.acc_cap);
    float *beta_sm = reinterpret_cast<float *>(red_d + (NORM ? MT * CWARPS : 0));
    uint32_t *red_u = reinterpret_cast<uint32_t *>(beta_sm + MT);   // [MT][CWARPS] absmax
    int *red_i = reinterpret_cast<int *>(red_u + MT * CWARPS);      // [MT][CWARPS] sum x~

    const int warp = threadIdx.x >> 5;
    const int lane = threadIdx.x & 31;
    const uint64_t limit = p.wait_limit_ns;

    if (threadIdx.x == 0) {
        for (int s = 0; s < slots; ++s) {
            mbar_init(full(s), 1);
            mbar_init(empty(s), CWARPS);
        }
        *abort_flag = 0;
        fence_barrier_init();
    }
    __syncthreads();

    if (warp == CWARPS) {
        // ---------------------------------------------------- weight producer
        // Reads only the packed weights, so it does not wait for the previous
        // grid in the stream.
        if (lane == 0) {
            int issued = 0;
            int slot = 0;
            uint32_t phase = 0;       // parity of this pass over the ring
            for (int st = 0; st < nstages; ++st) {
                // from the second pass on, the slot must have been released
                if (st >= slots && !mbar_wait_bounded(empty(slot), phase ^ 1u, abort_flag, limit))
                    break;
                const int off = st * STAGE;
                const int bytes = min(STAGE, npieces * PIECE - off);
                mbar_arrive_expect_tx(full(slot), static_cast<uint32_t>(bytes));
                bulk_g2s(smem_u32(ring + slot * STAGE), src + off, static_cast<uint32_t>(bytes),
                         full(slot));
                issued = st + 1;
                if (++slot == slots) {
                    slot = 0;
                    phase ^= 1u;
                }
            }
            // every copy this thread started lands before the block exits
            for (int st = max(0, issued - slots); st < issued; ++st)
                drain_wait(full(st % slots), static_cast<uint32_t>(st / slots) & 1u, limit);
        }
        return;
    }

    // ------------------------------------------------------- compute warps
    const int ctid = threadIdx.x;                       // 0 .. CTHREADS-1
    for (int i = ctid; i < nblk * 16 * MT; i += CTHREADS)
        acc_sm[i] = 0;

    // x may be the previous kernel's output: read it only after the wait.
    // Each thread keeps up to XCACHE vectors of 8 activations in registers
    // between the absmax pass and the quantisation pass; longer rows are read
    // again (from L1).
    pdl_wait();
    constexpr int XCACHE = 4;
    Vec8<BF16> xc[XCACHE];
    const int e0 = ctid * 8;
    const int estride = CTHREADS * 8;
    if constexpr (NORM) {
        // sums of squares per token (the first token's cache is filled here)
        for (int m = 0; m < M; ++m) {
            const void *row = static_cast<const char *>(P.x) +
                              static_cast<size_t>(m) * K * (BF16 ? 2 : 4);
            double ss = 0.0;
#pragma unroll
            for (int c = 0; c < XCACHE; ++c) {
                const int e = e0 + c * estride;
                if (m == 0 && e < K) {
                    xc[c].load(row, e);
#pragma unroll
                    for (int i = 0; i < 8; ++i) {
                        const double d = xc[c].get(i);
                        ss = __fma_rn(d, d, ss);
                    }
                }
            }
            for (int e = (m == 0 ? e0 + XCACHE * estride : e0); e < K; e += estride) {
                float v[8];
                load8<BF16>(row, e, v);
#pragma unroll
                for (int i = 0; i < 8; ++i) {
                    const double d = v[i];
                    ss = __fma_rn(d, d, ss);
                }
            }
            ss = warp_sum_f64(ss);
            if (lane == 0)
                red_d[m * CWARPS + warp] = ss;
        }
        compute_sync();
    }
    for (int m = 0; m < M; ++m) {
        const void *row = static_cast<const char *>(P.x) +
                          static_cast<size_t>(m) * K * (BF16 ? 2 : 4);
        float r = 1.0f;
        if constexpr (NORM)
            r = row_rms_scale(red_d, m, K, P.norm_eps);
        float amax = 0.0f;
#pragma unroll
        for (int c = 0; c < XCACHE; ++c) {
            const int e = e0 + c * estride;
            if (m == 0 && e < K) {
                float g[8];
                if constexpr (NORM)
                    load8<false>(P.norm_gain, e, g);
                else
                    xc[c].load(row, e);
#pragma unroll
                for (int i = 0; i < 8; ++i) {
                    float a = xc[c].get(i);
                    if constexpr (NORM)
                        a = norm1(a, r, g[i]);
                    amax = fmaxf(amax, fabsf(a));
                }
            }
        }
        for (int e = (m == 0 ? e0 + XCACHE * estride : e0); e < K; e += estride) {
            float v[8], g[8];
            load8<BF16>(row, e, v);
            if constexpr (NORM)
                load8<false>(P.norm_gain, e, g);
#pragma unroll
            for (int i = 0; i < 8; ++i) {
                float a = v[i];
                if constexpr (NORM)
                    a = norm1(a, r, g[i]);
                amax = fmaxf(amax, fabsf(a));
            }
        }
        const uint32_t u = __reduce_max_sync(0xffffffffu, __float_as_uint(amax));
        if (lane == 0)
            red_u[m * CWARPS + warp] = u;
    }
    compute_sync();
    for (int m = 0; m < M; ++m) {
        const void *row = static_cast<const char *>(P.x) +
                          static_cast<size_t>(m) * K * (BF16 ? 2 : 4);
        uint32_t u = red_u[m * CWARPS];
#pragma unroll
        for (int w = 1; w < CWARPS; ++w)
            u = max(u, red_u[m * CWARPS + w]);
        const float beta = fmaxf(__uint_as_float(u), 1e-5f);
        const float scale = __fdiv_rn(127.0f, beta);
        float r = 1.0f;
        if constexpr (NORM)
            r = row_rms_scale(red_d, m, K, P.norm_eps);
        int sum = 0;
        auto quant_store = [&](const Vec8<BF16> &v, int e) {
            float g[8];
            if constexpr (NORM)
                load8<false>(P.norm_gain, e, g);
            uint32_t lo = 0, hi = 0;
#pragma unroll
            for (int i = 0; i < 4; ++i) {
                float a = v.get(i), b = v.get(i + 4);
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
            *reinterpret_cast<uint2 *>(xq_sm + m * K + e) = make_uint2(lo, hi);
            if (P.xq_dbg != nullptr && blockIdx.x == 0)
                *reinterpret_cast<uint2 *>(P.xq_dbg + static_cast<size_t>(m) * K + e) =
                    make_uint2(lo, hi);
        };
        if (m == 0) {
#pragma unroll
            for (int c = 0; c < XCACHE; ++c) {
                const int e = e0 + c * estride;
                if (e < K)
                    quant_store(xc[c], e);
            }
        }
        for (int e = (m == 0 ? e0 + XCACHE * estride : e0); e < K; e += estride) {
            Vec8<BF16> v;
            v.load(row, e);
            quant_store(v, e);
        }
        sum = __reduce_add_sync(0xffffffffu, sum);
        if (lane == 0)
            red_i[m * CWARPS + warp] = sum;
        if (ctid == 0) {
            beta_sm[m] = beta;
            if (P.beta_dbg != nullptr && blockIdx.x == 0)
                P.beta_dbg[m] = beta;
        }
    }
    compute_sync();

    // ---- stream the pieces: piece i = (row block i / KG, k-group i % KG).
    // Warp w takes pieces w, w + CWARPS, ... of every stage: a fixed number
    // per stage, fully unrolled, with the (block, group) index of each piece
    // computed by a multiply-high instead of a division. Each piece's partial
    // dot product goes straight into the row accumulators, so the pieces of a
    // stage are independent and their loads and dp4a chains overlap.
    const int r = lane >> 1;          // row in the block
    const int t = lane & 1;           // k-half (64 weights) of the group
    // partial of one piece for token m: sum over its 64 weights of c * x~
    auto piece_dot = [&](const uint4 &w4, int gg, int m) -> int {
        const uint8_t *xk = xq_sm + m * K + gg * 128 + t * 64;
        const uint32_t words[4] = {w4.x, w4.y, w4.z, w4.w};
        int s1a = 0, s1b = 0, s4a = 0, s4b = 0;
#pragma unroll
        for (int jw = 0; jw < 4; ++jw) {
            const uint4 xv = *reinterpret_cast<const uint4 *>(xk + 16 * jw);
            const uint32_t w = words[jw], w_hi = w >> 4;
            // j = 0, 2 at scale 1; j = 1, 3 at scale 4
            if (jw & 1) {
                s1b = dp4a_ss(w & 0x03030303u, xv.x, s1b);
                s4b = dp4a_ss(w & 0x0C0C0C0Cu, xv.y, s4b);
                s1b = dp4a_ss(w_hi & 0x03030303u, xv.z, s1b);
                s4b = dp4a_ss(w_hi & 0x0C0C0C0Cu, xv.w, s4b);
            } else {
                s1a = dp4a_ss(w & 0x03030303u, xv.x, s1a);
                s4a = dp4a_ss(w & 0x0C0C0C0Cu, xv.y, s4a);
                s1a = dp4a_ss(w_hi & 0x03030303u, xv.z, s1a);
                s4a = dp4a_ss(w_hi & 0x0C0C0C0Cu, xv.w, s4a);
            }
        }
        return s1a + s1b + ((s4a + s4b) >> 2);
    };

    // The next kernel in the stream may start launching now: its weight
    // stream overlaps this main loop and epilogue.
    pdl_launch_dependents();

    int slot = 0;
    uint32_t phase = 0;
    for (int st = 0; st < nstages; ++st) {
        if (!warp_wait_bounded(full(slot), phase, abort_flag, limit))
            break;
        const uint8_t *stage = ring + slot * STAGE + lane * 16;
        const int pbase = st * PIECES_PER_STAGE;
        auto locate = [&](int local, int &b, int &gg) {
            const int i = pbase + local;
            b = static_cast<int>((static_cast<uint64_t>(i) * P.kg_magic) >> 32);
            gg = i - b * KG;
        };
        {
            // all of this warp's pieces of the slot at once, without branches;
            // the last slot may be short, and its missing pieces are computed
            // on stale slot bytes but not committed
            uint4 wv[PIECES_PER_WARP];
            int bv[PIECES_PER_WARP], gv[PIECES_PER_WARP];
            bool ok[PIECES_PER_WARP];
#pragma unroll
            for (int u = 0; u < PIECES_PER_WARP; ++u) {
                const int local = warp + CWARPS * u;
                ok[u] = pbase + local < npieces;
                wv[u] = *reinterpret_cast<const uint4 *>(stage + local * PIECE);
                locate(local, bv[u], gv[u]);
            }
#pragma unroll
            for (int m = 0; m < MT; ++m) {
                if (m < M) {
#pragma unroll
                    for (int u = 0; u < PIECES_PER_WARP; ++u) {
                        int v = piece_dot(wv[u], gv[u], m);
                        v += __shfl_xor_sync(0xffffffffu, v, 1);
                        if (t == 0 && ok[u])
                            atomicAdd(&acc_sm[(bv[u] * 16 + r) * MT + m], v);
                    }
                }
            }
        }
        __syncwarp();
        if (lane == 0)
            mbar_arrive(empty(slot));
        if (++slot == slots) {
            slot = 0;
            phase ^= 1u;
        }
    }
    compute_sync();

    // ---- epilogue: acc = sum c*x~ - sum x~, rescale, bf16
    for (int m = 0; m < M; ++m) {
        const float s = out_scale(beta_sm[m], P.gamma);
        int rs = 0;
#pragma unroll
        for (int w = 0; w < CWARPS; ++w)
            rs += red_i[m * CWARPS + w];
        for (int rl = ctid; rl < nblk * 16; rl += CTHREADS) {
            const int n = blk0 * 16 + rl;
            if (n < N) {
                const int a = acc_sm[rl * MT + m] - rs;
                const size_t o = static_cast<size_t>(m) * N + n;
                P.y[o] = rescale_bf16(a, s);
                if (P.acc_dbg != nullptr)
                    P.acc_dbg[o] = a;
            }
        }
    }
}

}  // namespace gemv
}  // namespace bitlinear
