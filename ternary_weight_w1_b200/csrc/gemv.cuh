// Decode GEMV for small M: y = BitLinear(x) with the activation quantisation
// fused in the prologue and the packed ternary weights streamed from HBM once.
//
// Pages: "BitNet b1.58 2B4T Guide: Scaling Native 1-Bit LLMs", sections
// "8-Bit Activation Quantization: absmax Scaling" (prologue), "Matrix
// Multiplication as Pure Integer Addition" (contraction and rescale); the
// memory-wall framing of "BitNet b1.58: The 1-Bit Paradigm Shift" is why the
// kernel is organised around the weight bytes.
//
// Work split. The packed layout keeps 16-row blocks contiguous, each block a
// run of K/128 512-byte pieces (one 128-k group of its 16 rows). CTA c owns
// q consecutive row blocks of one problem and takes them in chunks of up to
// QB blocks. A chunk is streamed k-group-major: stage s holds groups
// [G s, G s + G) of every block of the chunk, one bulk copy per block issued
// by its own producer lane, all landing on the stage's mbarrier. The producer
// starts before the programmatic-launch wait (the weights are never written
// by an earlier kernel), so the stream overlaps the previous kernel and this
// kernel's prologue.
//
// Compute warp w owns the k-groups g = w (mod 8). In a stage it loads, for
// each of its groups, the 64 bytes of x~ its lane needs into registers once
// and applies them to that group's piece of every block of the chunk: lane
// (r, t) = (lane / 2, lane % 2) holds row r of the block and the k-half t of
// the group (64 weights, 16 bytes). The row partial sums stay in registers
// for the whole chunk; one shuffle (the two k-halves) and one pass through
// shared memory (the eight warps) per chunk give the rows' sums.
//
// Arithmetic. With codes c = W~ + 1 in {0, 1, 2} at bits 2j of every byte of
// a packed word, w & (3 << 2j) leaves c * 4^j in each byte (at most 128,
// which fits an unsigned byte), so one dp4a of unsigned weight bytes by
// signed x~ bytes per plane and token multiplies four weights by the matching
// x~ word. The plane sums a_j are exact multiples of 4^j, so
//   sum c * x~ = a_0 + (a_1 >> 2) + (a_2 >> 4) + (a_3 >> 6)
// exactly, and acc = sum c * x~ - sum x~. Integer sums: the order of the
// partial sums cannot change the result.
//
// Prologue. Each thread reads the activations of its own warp's groups in
// 16-byte slots (half-warp h: group w + 8 (2 i + h), lane l: elements
// 128 g + 8 (l % 16) .. + 7), keeping the first slots of token 0 in
// registers between the passes; the warps combine their absmax through
// shared memory (one barrier; for bf16 the maximum of the 15-bit magnitude
// fields, two per word, which orders finite values as |x| does), and every
// warp quantises its own groups into shared memory, where only its own lanes
// read them. The sum of x~ of each
// warp's groups goes to shared memory for the epilogue. With RMS
// normalisation (NORM launches; the listing's BitLinear normalises each token
// with its nn.RMSNorm member before quantising it) a first pass sums each
// token's squares in double (exact products), the warps' sums go to shared
// memory and every thread adds them in warp order, so all CTAs derive the
// same r = 1 / sqrt(mean + eps); the absmax and quantisation passes then work
// on (x * r) * g.
//
// Feed-forward form (FFN launches). The gate and up projections of a
// feed-forward block read the same tokens: a CTA streams block b of both
// matrices in the same stage (gate blocks in the first half of the slot, up
// blocks in the second), applies the same x~ registers to both (or, when
// each projection RMS-normalises the tokens with its own gains, its own x~),
// and its epilogue rounds both outputs to bf16 and writes the gated squared
// ReLU h = (r * r) * up, r = max(gate, 0), in fp32: the feed-forward
// activation of "Microsoft Releases BitNet b1.58 2B4T" ("Under the Hood":
// ReLU^2 in place of SwiGLU), read as gated. h is the down projection's input.
//
// Every mbarrier wait is bounded; a wait that runs out records the fault
// word, raises the block's abort flag so that every warp stops waiting, and
// the epilogue then writes nothing (no partial y). The producer waits for its
// own copies before it returns.
#pragma once

#include "common.cuh"

namespace bitlinear {
namespace gemv {

constexpr int CWARPS = 8;                          // compute warps
constexpr int CTHREADS = CWARPS * 32;
constexpr int THREADS = CTHREADS + 32;             // + the producer warp
constexpr int PIECE = 512;                         // one (row block, k-group)
constexpr int MAX_SLOTS = 8;
constexpr int BAR_BYTES = 2 * MAX_SLOTS * 8 + 16;  // full/empty barriers + abort flag
constexpr int MAX_PROBLEMS = 8;
// 16-byte slots of token 0 kept in registers through the prologue (a warp's
// share of K <= 8192)
constexpr int XCACHE = 4;

// Row blocks per chunk and tokens whose x~ a lane holds in registers at once,
// by token tile MT. Only MT = 1 keeps the four plane sums apart for a whole
// chunk; larger tiles fold them into one sum per piece.
template <int MT, bool FFN = false>
struct Shape {
    // an FFN chunk carries each block twice (gate and up)
    static constexpr int QB = (MT == 1 ? 8 : MT == 2 ? 4 : 2) / (FFN ? 2 : 1);
    static constexpr int TQ = MT == 4 ? 4 : MT == 1 ? 1 : 2;
    static constexpr bool PERSIST = MT == 1;
    // blocks per SM the register budget is set for: three for the small
    // tiles (two of this launch and, under programmatic dependent launch, one
    // of the next), two for the larger ones and the normalising forms
    static constexpr int MIN_BLOCKS = (MT <= 2 && !FFN) ? 3 : 2;
};

__host__ __device__ constexpr int chunk_blocks(int MT, bool ffn = false)
{
    return (MT == 1 ? 8 : MT == 2 ? 4 : 2) / (ffn ? 2 : 1);
}

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
    int base, extra;        // row blocks of 16 rows per CTA: base, one more for the
                            // problem's first `extra` CTAs
    int cta_begin;          // this problem's first CTA in the grid
    int cb;                 // row blocks per chunk (<= QB)
    int G;                  // k-groups per stage (a multiple of 8, or all K/128: then a
                            // stage is whole rows, one contiguous copy per matrix)
    // FFN launches only: `packed`, `gamma`, `norm_gain` and `y` (optional)
    // are the gate projection's; these are the up projection's and h
    const uint8_t *packed2;
    float gamma2;
    const float *norm_gain2;
    uint16_t *y2;           // [M][N] bf16 up output, or null
    float *h;               // [M][N] fp32 (r * r) * up, r = max(gate, 0)
};

struct Params {
    Problem prob[MAX_PROBLEMS];
    int count;              // problems in this launch
    int slots;              // ring slots (<= MAX_SLOTS)
    int slot_bytes;         // bytes per ring slot (a multiple of 512)
    int xq_cap;             // shared bytes for x~: max over problems of M * K
    int red_blocks;         // row blocks per chunk the reduction area holds
    uint64_t wait_limit_ns;
    int inject_timeout;     // the producer leaves the first stage unloaded
};

// Shared-memory bytes of a launch (the regions in the order the kernel
// carves them out; every region size is a multiple of 16 bytes). An FFN
// launch keeps two reduction areas (gate and up) and, when it normalises,
// two quantised copies of the tokens with their own beta and sums.
// A base-3 launch adds its 256-entry decoding table.
__host__ __device__ constexpr int smem_bytes(int MT, int xq_cap, int slots, int slot_bytes,
                                             int red_blocks, bool norm, bool ffn = false,
                                             bool b3 = false)
{
    return slots * slot_bytes + BAR_BYTES + (ffn && norm ? 2 : 1) * xq_cap +
           (ffn ? 2 : 1) * CWARPS * red_blocks * 16 * MT * 4 + (norm ? MT * CWARPS * 8 : 0) +
           (ffn && norm ? 2 : 1) * (16 * ((MT * 4 + 15) / 16) + 2 * MT * CWARPS * 4) +
           (b3 ? 256 * 4 : 0);
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

// dp4a of four unsigned bytes (weight codes times a power of 4, at most 128)
// by four signed bytes (x~), accumulated in int32.
__device__ __forceinline__ int dp4a_us(uint32_t a, uint32_t b, int c)
{
    int d;
    asm("dp4a.u32.s32 %0, %1, %2, %3;" : "=r"(d) : "r"(a), "r"(b), "r"(c));
    return d;
}

// Four consecutive activations (element e, a multiple of 4) of a row as fp32
// (bf16 widening is exact).
template <bool BF16>
__device__ __forceinline__ void load4(const void *row, int e, float (&v)[4])
{
    if constexpr (BF16) {
        const uint2 raw =
            __ldg(reinterpret_cast<const uint2 *>(static_cast<const __nv_bfloat16 *>(row) + e));
        v[0] = __uint_as_float(raw.x << 16);
        v[1] = __uint_as_float(raw.x & 0xffff0000u);
        v[2] = __uint_as_float(raw.y << 16);
        v[3] = __uint_as_float(raw.y & 0xffff0000u);
    } else {
        const float4 a = __ldg(reinterpret_cast<const float4 *>(static_cast<const float *>(row) + e));
        v[0] = a.x; v[1] = a.y; v[2] = a.z; v[3] = a.w;
    }
}

// WIDE (one bf16 token of 8192 < K <= 32768, no normalisation, not FFN)
// stages the token row in shared memory for the prologue (two blocks per SM).
// B3 reads the base-3 layout (five codes per byte; no normalisation, not FFN,
// not WIDE): a 256-entry table in shared memory turns each byte back into ten
// bits of 2-bit codes, rebuilding the 2-bit layout's words in registers.
template <int MT, bool BF16, bool NORM, bool FFN, bool WIDE, bool B3 = false>
__global__ void __launch_bounds__(THREADS,
                                  ((NORM || WIDE || B3) ? 2 : Shape<MT, FFN>::MIN_BLOCKS))
gemv_kernel(const __grid_constant__ Params p)
{
    using S = Shape<MT, FFN>;
    constexpr int QB = S::QB;
    constexpr int NMAT = FFN ? 2 : 1;          // matrices streamed (gate, up)
    constexpr int NX = (FFN && NORM) ? 2 : 1;   // quantised copies of the tokens
    // with two copies of x~ in registers, fewer tokens at a time
    // (and with the base-3 layout's five-word x~ runs)
    constexpr int TQ = (NX == 1 && !B3) ? S::TQ : MT >= 8 ? 1 : (S::TQ < 2 ? S::TQ : 2);
    constexpr int NACC = S::PERSIST ? 4 : MT;   // accumulators per block and matrix
    extern __shared__ __align__(128) uint8_t smem[];
    // this CTA's problem (grouped launches give each problem its own CTAs)
    int pi = 0;
#pragma unroll 1
    while (pi + 1 < p.count && static_cast<int>(blockIdx.x) >= p.prob[pi + 1].cta_begin)
        ++pi;
    const Problem &P = p.prob[pi];
    const int K = P.K, M = P.M, N = P.N;
    // k-groups per row: of 128 weights, or of 160 in the base-3 layout, whose
    // rows (and x~ rows) are padded to XS = 160 KG
    constexpr int GW = B3 ? 160 : 128;                  // weights per k-group
    constexpr int NW = GW / 32;                         // code words per lane and piece
    const int KG = B3 ? (K + 159) / 160 : K >> 7;
    const int XS = B3 ? KG * 160 : K;
    const int G = P.G;
    const int total_blocks = (N + 15) >> 4;
    const int cta = static_cast<int>(blockIdx.x) - P.cta_begin;
    const int blk0 = cta * P.base + min(cta, P.extra);
    const int nblk = min(P.base + (cta < P.extra ? 1 : 0), total_blocks - blk0);
    const int cb = P.cb;
    const int nchunks = (nblk + cb - 1) / cb;
    const int kstages = (KG + G - 1) / G;
    const int nstages = nchunks * kstages;
    const int slots = p.slots;
    const int slot_bytes = p.slot_bytes;
    const int red_stride = CWARPS * p.red_blocks * 16 * MT;     // ints per reduction area
    const bool first_cta = static_cast<int>(blockIdx.x) == P.cta_begin;

    uint8_t *ring = smem;
    const uint32_t ring_u32 = smem_u32(ring);
    const uint32_t bars = smem_u32(smem + slots * slot_bytes);
    auto full = [&](int s) { return bars + 8u * static_cast<uint32_t>(s); };
    auto empty = [&](int s) { return bars + 8u * static_cast<uint32_t>(MAX_SLOTS + s); };
    volatile int *abort_flag =
        reinterpret_cast<volatile int *>(smem + slots * slot_bytes + 2 * MAX_SLOTS * 8);
    uint8_t *xq_sm = smem + slots * slot_bytes + BAR_BYTES;        // [NX][xq_cap]
    int *red = reinterpret_cast<int *>(xq_sm + NX * p.xq_cap);      // [NMAT][CWARPS][blocks*16][MT]
    // [MT][CWARPS] partial sums of squares (NORM only; 8-byte aligned: every
    // region before it is a multiple of 16 bytes)
    double *red_d = reinterpret_cast<double *>(red + NMAT * red_stride);
    // per quantised copy: beta [MT (rounded up to 4)], absmax and sum of x~
    // partials [MT][CWARPS]
    constexpr int QSET = 4 * ((MT + 3) / 4) + 2 * MT * CWARPS;
    float *qset = reinterpret_cast<float *>(red_d + (NORM ? MT * CWARPS : 0));
    auto beta_sm = [&](int x) { return qset + x * QSET; };
    auto red_u = [&](int x) { return reinterpret_cast<uint32_t *>(qset + x * QSET + 4 * ((MT + 3) / 4)); };
    auto red_s = [&](int x) { return reinterpret_cast<int *>(red_u(x) + MT * CWARPS); };
    // base-3 decoding table: byte value -> its five codes as 2-bit fields
    uint32_t *lut = reinterpret_cast<uint32_t *>(qset + NX * QSET);

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
    if constexpr (B3) {
        // entry v: the base-3 digits of v (0 .. 242) as 2-bit codes at bits
        // 2i; bytes above 242 do not occur and decode to zero weights
        for (int v = threadIdx.x; v < 256; v += THREADS) {
            uint32_t f = 0x155u;
            if (v < 243) {
                f = 0;
                int t = v;
                for (int i = 0; i < 5; ++i) {
                    f |= static_cast<uint32_t>(t % 3) << (2 * i);
                    t /= 3;
                }
            }
            lut[v] = f;
        }
    }
    __syncthreads();
    // The next kernel in the stream may start launching at once: its CTAs
    // take the SMs' free slots and start their weight streams while this
    // launch runs (they wait for it to complete before reading its outputs).
    pdl_launch_dependents();

    if (warp == CWARPS) {
        // ---------------------------------------------------- weight producer
        // Reads only the packed weights, so it does not wait for the previous
        // grid in the stream. A stage of whole rows is one copy per matrix
        // (lane 1: the up projection's rows of an FFN launch); a stage of a
        // k-range takes lane l for block l of the chunk (FFN: lanes qb ..
        // 2 qb - 1 for the up projection). Lane 0 arms the stage's barrier with
        // the whole stage's bytes first.
        int slot = 0;
        uint32_t phase = 0;        // parity of this pass over the ring
        uint32_t in_flight = 0;    // slots holding a copy this warp issued
        uint32_t parity = 0;       // the phase of that copy, per slot
        for (int st = 0; st < nstages; ++st) {
            // from the second pass on, the slot must have been released
            if (st >= slots &&
                !warp_wait_sleep_bounded(empty(slot), phase ^ 1u, abort_flag, limit))
                break;
            const int c = st / kstages;
            const int ks = st - c * kstages;
            const int b0 = c * cb;
            const int qb = min(cb, nblk - b0);
            const int g0 = ks * G;
            const int gs = min(G, KG - g0);
            const uint32_t bytes = static_cast<uint32_t>(gs * PIECE);
            // the failure-detection test leaves the first stage unloaded, so
            // the compute warps' first wait runs out
            if (!(p.inject_timeout && st == 0)) {
                if (lane == 0)
                    mbar_arrive_expect_tx(full(slot), bytes * static_cast<uint32_t>(NMAT * qb));
                __syncwarp();
                if (gs == KG) {
                    // whole rows: the chunk's blocks are one contiguous range
                    // per matrix
                    if (lane < NMAT) {
                        const uint8_t *src = (FFN && lane == 1) ? P.packed2 : P.packed;
                        bulk_g2s(ring_u32 + static_cast<uint32_t>(slot * slot_bytes) +
                                     lane * qb * bytes,
                                 src + static_cast<size_t>(blk0 + b0) * KG * PIECE,
                                 bytes * static_cast<uint32_t>(qb), full(slot));
                    }
                } else if (lane < NMAT * qb) {
                    // a k-range of every block: one copy per block
                    const int mat = lane >= qb ? 1 : 0;
                    const int bl = lane - mat * qb;
                    const uint8_t *src = (FFN && mat) ? P.packed2 : P.packed;
                    bulk_g2s(ring_u32 + static_cast<uint32_t>(slot * slot_bytes) + lane * bytes,
                             src + (static_cast<size_t>(blk0 + b0 + bl) * KG + g0) * PIECE, bytes,
                             full(slot));
                }
                in_flight |= 1u << slot;
                parity = (parity & ~(1u << slot)) | (phase << slot);
            }
            if (++slot == slots) {
                slot = 0;
                phase ^= 1u;
            }
        }
        // every copy this warp started lands before the block exits
        if (lane == 0)
            for (int s = 0; s < slots; ++s)
                if (in_flight & (1u << s))
                    drain_wait(full(s), (parity >> s) & 1u, limit);
        __syncwarp();
        return;
    }

    // ------------------------------------------------------- compute warps
    const int ctid = threadIdx.x;                       // 0 .. CTHREADS-1
    const size_t row_bytes = static_cast<size_t>(K) * (BF16 ? 2 : 4);
    const int ngw = (KG - warp + CWARPS - 1) / CWARPS;  // this warp's groups: warp + 8 i

    // x may be the previous kernel's output: read it only after the wait.
    pdl_wait();
    // Slot i of this thread: group g = warp + 8 (2 i + h), h = lane / 16 (two
    // of this warp's groups per slot), elements 128 g + 8 (lane % 16) .. + 7,
    // one 16-byte load of bf16 (two of fp32). Token 0's first XCACHE slots
    // stay in registers between the passes; the rest are read again, XB
    // slots at a time so that their loads are in flight together.
    const int h = lane >> 4;
    auto slot_group = [&](int i) { return warp + CWARPS * (2 * i + h); };
    auto slot_elem = [&](int i) { return slot_group(i) * 128 + 8 * (lane & 15); };
    const int nsl = (ngw + 1) / 2;                    // slots of this warp
    // gains of quantised copy x (FFN: 0 = gate, 1 = up)
    auto gain_of = [&](int x) { return (FFN && x == 1) ? P.norm_gain2 : P.norm_gain; };
    if constexpr (B3) {
        // The base-3 layout pads each row to XS = 160 KG weights: the tokens
        // are quantised by all compute threads together into x~ rows of XS
        // bytes whose padding is zero, and a block barrier makes them visible
        // to every warp.
        static_assert(!NORM && !FFN && !WIDE, "base-3 kernel");
        for (int m = 0; m < M; ++m) {
            const void *row = static_cast<const char *>(P.x) + m * row_bytes;
            float amax = 0.0f;
            for (int e = ctid * 8; e < K; e += CTHREADS * 8) {
                Vec8<BF16> v;
                v.load(row, e);
#pragma unroll
                for (int u = 0; u < 8; ++u)
                    amax = fmaxf(amax, fabsf(v.get(u)));
            }
            const uint32_t um = __reduce_max_sync(0xffffffffu, __float_as_uint(amax));
            if (lane == 0)
                red_u(0)[m * CWARPS + warp] = um;
        }
        compute_sync();
        for (int m = 0; m < M; ++m) {
            const void *row = static_cast<const char *>(P.x) + m * row_bytes;
            uint32_t ub = red_u(0)[m * CWARPS];
#pragma unroll
            for (int w = 1; w < CWARPS; ++w)
                ub = max(ub, red_u(0)[m * CWARPS + w]);
            const float beta = fmaxf(__uint_as_float(ub), 1e-5f);
            const float scale = __fdiv_rn(127.0f, beta);
            int sum = 0;
            for (int e = ctid * 8; e < XS; e += CTHREADS * 8) {
                uint32_t lo = 0, hi = 0;
                if (e < K) {
                    Vec8<BF16> v;
                    v.load(row, e);
                    // |x * (127 / beta)| <= 127: the listing's clamp cannot bind
                    uint32_t q[8];   // rint(x * scale) in the low byte (rint_bits)
#pragma unroll
                    for (int u = 0; u < 8; ++u)
                        q[u] = rint_bits(__fmul_rn(v.get(u), scale));
                    lo = __byte_perm(__byte_perm(q[0], q[1], 0x0040),
                                     __byte_perm(q[2], q[3], 0x0040), 0x5410);
                    hi = __byte_perm(__byte_perm(q[4], q[5], 0x0040),
                                     __byte_perm(q[6], q[7], 0x0040), 0x5410);
                    sum = dp4a_ss(hi, 0x01010101u, dp4a_ss(lo, 0x01010101u, sum));
                    if (P.xq_dbg != nullptr && first_cta)
                        *reinterpret_cast<uint2 *>(P.xq_dbg + static_cast<size_t>(m) * K + e) =
                            make_uint2(lo, hi);
                }
                *reinterpret_cast<uint2 *>(xq_sm + m * XS + e) = make_uint2(lo, hi);
            }
            sum = __reduce_add_sync(0xffffffffu, sum);
            if (lane == 0)
                red_s(0)[m * CWARPS + warp] = sum;
            if (ctid == 0) {
                beta_sm(0)[m] = beta;
                if (P.beta_dbg != nullptr && first_cta)
                    P.beta_dbg[m] = beta;
            }
        }
        compute_sync();
    } else if constexpr (WIDE) {
        // One bf16 token of up to 32768 activations. Its row is staged in
        // shared memory (the 2 K bytes of the x~ region, which x~ overwrites
        // at the end) with 16-byte asynchronous copies of every slot of this
        // thread, all in flight at once; both passes then read shared memory,
        // and the quantised words wait in registers until every thread has
        // read its slots.
        static_assert(BF16 && !NORM && !FFN && MT == 1, "wide kernel");
        constexpr int WSL = 16;                       // slots per thread at K = 32768
        const char *row = static_cast<const char *>(P.x);
        auto valid = [&](int i) { return i < nsl && slot_group(i) < KG; };
#pragma unroll
        for (int i = 0; i < WSL; ++i)
            if (valid(i))
                cp_async16(smem_u32(xq_sm + 2 * slot_elem(i)), row + 2 * slot_elem(i));
        cp_async_wait_all();
        auto staged = [&](int i) {
            Vec8<true> v;
            const uint4 raw = *reinterpret_cast<const uint4 *>(xq_sm + 2 * slot_elem(i));
            v.w[0] = raw.x; v.w[1] = raw.y; v.w[2] = raw.z; v.w[3] = raw.w;
            return v;
        };
        float amax = 0.0f;
#pragma unroll
        for (int i = 0; i < WSL; ++i) {
            if (valid(i)) {
                const Vec8<true> v = staged(i);
#pragma unroll
                for (int u = 0; u < 8; ++u)
                    amax = fmaxf(amax, fabsf(v.get(u)));
            }
        }
        const uint32_t um = __reduce_max_sync(0xffffffffu, __float_as_uint(amax));
        if (lane == 0)
            red_u(0)[warp] = um;
        compute_sync();
        uint32_t ub = red_u(0)[0];
#pragma unroll
        for (int w = 1; w < CWARPS; ++w)
            ub = max(ub, red_u(0)[w]);
        const float beta = fmaxf(__uint_as_float(ub), 1e-5f);
        const float scale = __fdiv_rn(127.0f, beta);
        uint32_t qw[WSL][2];
        int sum = 0;
#pragma unroll
        for (int i = 0; i < WSL; ++i) {
            if (valid(i)) {
                const Vec8<true> v = staged(i);
                // |x * (127 / beta)| <= 127: the listing's clamp cannot bind
                uint32_t q[8];   // rint(x * scale) in the low byte (rint_bits)
#pragma unroll
                for (int u = 0; u < 8; ++u)
                    q[u] = rint_bits(__fmul_rn(v.get(u), scale));
                qw[i][0] = __byte_perm(__byte_perm(q[0], q[1], 0x0040),
                                       __byte_perm(q[2], q[3], 0x0040), 0x5410);
                qw[i][1] = __byte_perm(__byte_perm(q[4], q[5], 0x0040),
                                       __byte_perm(q[6], q[7], 0x0040), 0x5410);
                sum = dp4a_ss(qw[i][1], 0x01010101u, dp4a_ss(qw[i][0], 0x01010101u, sum));
            }
        }
        // every thread has read its staged slots before x~ overwrites them
        compute_sync();
#pragma unroll
        for (int i = 0; i < WSL; ++i) {
            if (valid(i)) {
                const int e = slot_elem(i);
                *reinterpret_cast<uint2 *>(xq_sm + e) = make_uint2(qw[i][0], qw[i][1]);
                if (P.xq_dbg != nullptr && first_cta)
                    *reinterpret_cast<uint2 *>(P.xq_dbg + e) = make_uint2(qw[i][0], qw[i][1]);
            }
        }
        sum = __reduce_add_sync(0xffffffffu, sum);
        if (lane == 0)
            red_s(0)[warp] = sum;
        if (ctid == 0) {
            beta_sm(0)[0] = beta;
            if (P.beta_dbg != nullptr && first_cta)
                P.beta_dbg[0] = beta;
        }
    } else {
        Vec8<BF16> xc[XCACHE];
        // slots whose loads are issued together, and gain loads of cached slots
        constexpr int XB = NORM ? 2 : (BF16 ? 4 : 2);
        constexpr int XG = NORM ? 2 : XCACHE;
        using Gains = float[NX][8];
        // Visits this thread's valid slots of token m: f(i, v, g) with v the eight
        // raw activations and, when `gains` is set (NORM launches), g the eight
        // gains of each quantised copy.
        auto for_slots = [&](int m, bool fill, bool gains, auto &&f) {
            const void *row = static_cast<const char *>(P.x) + m * row_bytes;
            auto valid = [&](int i) { return i < nsl && slot_group(i) < KG; };
            auto load_gains = [&](int i, Gains &g) {
                if constexpr (NORM) {
                    if (gains) {
    #pragma unroll
                        for (int x = 0; x < NX; ++x)
                            load8<false>(gain_of(x), slot_elem(i), g[x]);
                    }
                }
            };
            int i0 = 0;
            if (m == 0) {
                if (fill) {
    #pragma unroll
                    for (int i = 0; i < XCACHE; ++i)
                        if (valid(i))
                            xc[i].load(row, slot_elem(i));
                }
    #pragma unroll
                for (int ic = 0; ic < XCACHE; ic += XG) {
                    float g[XG][NX][8];
    #pragma unroll
                    for (int u = 0; u < XG; ++u)
                        if (valid(ic + u))
                            load_gains(ic + u, g[u]);
    #pragma unroll
                    for (int u = 0; u < XG; ++u)
                        if (valid(ic + u))
                            f(ic + u, xc[ic + u], g[u]);
                }
                i0 = XCACHE;
            }
            for (int ib = i0; ib < nsl; ib += XB) {
                Vec8<BF16> v[XB];
                float g[XB][NX][8];
    #pragma unroll
                for (int u = 0; u < XB; ++u) {
                    if (valid(ib + u)) {
                        v[u].load(row, slot_elem(ib + u));
                        load_gains(ib + u, g[u]);
                    }
                }
    #pragma unroll
                for (int u = 0; u < XB; ++u)
                    if (valid(ib + u))
                        f(ib + u, v[u], g[u]);
            }
        };

        if constexpr (NORM) {
            // sums of squares per token
            for (int m = 0; m < M; ++m) {
                double ss = 0.0;
                for_slots(m, true, false, [&](int, const Vec8<BF16> &v, const Gains &) {
    #pragma unroll
                    for (int u = 0; u < 8; ++u) {
                        const double d = v.get(u);
                        ss = __fma_rn(d, d, ss);
                    }
                });
                ss = warp_sum_f64(ss);
                if (lane == 0)
                    red_d[m * CWARPS + warp] = ss;
            }
            compute_sync();
        }
        // absmax per token over this thread's elements (per quantised copy)
        for (int m = 0; m < M; ++m) {
            float r = 1.0f;
            if constexpr (NORM)
                r = row_rms_scale(red_d, m, K, P.norm_eps);
            float amax[NX];
    #pragma unroll
            for (int x = 0; x < NX; ++x)
                amax[x] = 0.0f;
            if constexpr (BF16 && !NORM) {
                // |x| of a finite bf16 orders like its bit pattern with the
                // sign cleared: the maximum of those 15-bit fields, two per
                // word, is the absmax (widened exactly at the end)
                uint32_t mb = 0;
                for_slots(m, true, false, [&](int, const Vec8<BF16> &v, const Gains &) {
    #pragma unroll
                    for (int j = 0; j < 4; ++j)
                        mb = max_u16x2(mb, v.w[j] & 0x7fff7fffu);
                });
                amax[0] = __uint_as_float(max(mb & 0xffffu, mb >> 16) << 16);
            } else {
                for_slots(m, !NORM, true, [&](int, const Vec8<BF16> &v, const Gains &g) {
    #pragma unroll
                    for (int x = 0; x < NX; ++x) {
    #pragma unroll
                        for (int u = 0; u < 8; ++u) {
                            float a = v.get(u);
                            if constexpr (NORM)
                                a = norm1(a, r, g[x][u]);
                            amax[x] = fmaxf(amax[x], fabsf(a));
                        }
                    }
                });
            }
    #pragma unroll
            for (int x = 0; x < NX; ++x) {
                const uint32_t u = __reduce_max_sync(0xffffffffu, __float_as_uint(amax[x]));
                if (lane == 0)
                    red_u(x)[m * CWARPS + warp] = u;
            }
        }
        compute_sync();
        // quantise this warp's own groups into shared memory (only this warp
        // reads them), with their sums of x~
        for (int m = 0; m < M; ++m) {
            float r = 1.0f;
            if constexpr (NORM)
                r = row_rms_scale(red_d, m, K, P.norm_eps);
            float scale[NX];
            int sum[NX];
    #pragma unroll
            for (int x = 0; x < NX; ++x) {
                uint32_t ub = red_u(x)[m * CWARPS];
    #pragma unroll
                for (int w = 1; w < CWARPS; ++w)
                    ub = max(ub, red_u(x)[m * CWARPS + w]);
                const float beta = fmaxf(__uint_as_float(ub), 1e-5f);
                scale[x] = __fdiv_rn(127.0f, beta);
                sum[x] = 0;
                if (ctid == 0) {
                    beta_sm(x)[m] = beta;
                    if (x == 0 && P.beta_dbg != nullptr && first_cta)
                        P.beta_dbg[m] = beta;
                }
            }
            for_slots(m, false, true, [&](int i, const Vec8<BF16> &v, const Gains &g) {
                const int e = slot_elem(i);
    #pragma unroll
                for (int x = 0; x < NX; ++x) {
                    // |a * (127 / beta)| <= 127 (beta is the row's absmax, or
                    // 1e-5 above every |a|), so rint never leaves [-127, 127]
                    // and the listing's clamp to [-128, 127] cannot bind
                    uint32_t q[8];   // rint(x * scale) in the low byte (rint_bits)
    #pragma unroll
                    for (int u = 0; u < 8; ++u) {
                        float a = v.get(u);
                        if constexpr (NORM)
                            a = norm1(a, r, g[x][u]);
                        q[u] = rint_bits(__fmul_rn(a, scale[x]));
                    }
                    const uint32_t lo = __byte_perm(__byte_perm(q[0], q[1], 0x0040),
                                                    __byte_perm(q[2], q[3], 0x0040), 0x5410);
                    const uint32_t hi = __byte_perm(__byte_perm(q[4], q[5], 0x0040),
                                                    __byte_perm(q[6], q[7], 0x0040), 0x5410);
                    sum[x] = dp4a_ss(hi, 0x01010101u, dp4a_ss(lo, 0x01010101u, sum[x]));
                    *reinterpret_cast<uint2 *>(xq_sm + x * p.xq_cap + m * K + e) = make_uint2(lo, hi);
                    if (x == 0 && P.xq_dbg != nullptr && first_cta)
                        *reinterpret_cast<uint2 *>(P.xq_dbg + static_cast<size_t>(m) * K + e) =
                            make_uint2(lo, hi);
                }
            });
    #pragma unroll
            for (int x = 0; x < NX; ++x) {
                const int sm = __reduce_add_sync(0xffffffffu, sum[x]);
                if (lane == 0)
                    red_s(x)[m * CWARPS + warp] = sm;
            }
        }
    }
    // this warp's lanes read the groups its lanes just wrote
    __syncwarp();

    const int r = lane >> 1;          // row in the block
    const int t = lane & 1;           // k-half (64 weights) of the group
    int slot = 0;
    uint32_t phase = 0;
    bool ok = true;
    for (int c = 0; c < nchunks; ++c) {
        const int b0 = c * cb;
        const int qb = min(cb, nblk - b0);
        // acc[mat][bi][.]: row sums of this lane's weights (PERSIST: the four
        // plane sums of token 0 kept apart, combined at the end of the chunk)
        int acc[NMAT][QB][NACC];
#pragma unroll
        for (int mat = 0; mat < NMAT; ++mat)
#pragma unroll
            for (int bi = 0; bi < QB; ++bi)
#pragma unroll
                for (int j = 0; j < NACC; ++j)
                    acc[mat][bi][j] = 0;

        for (int ks = 0; ks < kstages; ++ks) {
            if (ok)
                ok = warp_wait_sleep_bounded(full(slot), phase, abort_flag, limit);
            if (ok) {
                const int g0 = ks * G;
                const int gs = min(G, KG - g0);
                const uint8_t *stage = ring + slot * slot_bytes + lane * 16;
                for (int gi = warp; gi < gs; gi += CWARPS) {
#pragma unroll
                    for (int m0 = 0; m0 < MT; m0 += TQ) {
                        if (m0 < M) {
                            // x~ of this lane's GW / 2 weights for tokens m0 .. m0+TQ-1
                            uint32_t X[NX][TQ][4 * NW];
#pragma unroll
                            for (int x = 0; x < NX; ++x) {
                                const uint8_t *xg =
                                    xq_sm + x * p.xq_cap + (g0 + gi) * GW + t * (GW / 2);
#pragma unroll
                                for (int mq = 0; mq < TQ; ++mq) {
#pragma unroll
                                    for (int v = 0; v < NW; ++v) {
                                        // tokens past M (a smaller problem of a
                                        // grouped launch) read nothing
                                        const uint4 xv = (m0 + mq < M)
                                                             ? *reinterpret_cast<const uint4 *>(
                                                                   xg + (m0 + mq) * XS + 16 * v)
                                                             : make_uint4(0, 0, 0, 0);
                                        X[x][mq][4 * v] = xv.x; X[x][mq][4 * v + 1] = xv.y;
                                        X[x][mq][4 * v + 2] = xv.z; X[x][mq][4 * v + 3] = xv.w;
                                    }
                                }
                            }
#pragma unroll
                            for (int mat = 0; mat < NMAT; ++mat) {
                                constexpr int XL = NX - 1;
                                const int xs = mat < NX ? mat : XL;   // the copy this matrix reads
#pragma unroll
                                for (int bi = 0; bi < QB; ++bi) {
                                    if (bi >= qb)
                                        break;
                                    {
                                        const uint4 w4 = *reinterpret_cast<const uint4 *>(
                                            stage + ((mat * qb + bi) * gs + gi) * PIECE);
                                        uint32_t wd[NW];
                                        if constexpr (B3) {
                                            // byte B of the lane's 16 holds the
                                            // 2-bit fields 5B .. 5B+4 of its
                                            // five-word code stream
                                            const uint32_t by[4] = {w4.x, w4.y, w4.z, w4.w};
#pragma unroll
                                            for (int q = 0; q < NW; ++q)
                                                wd[q] = 0;
#pragma unroll
                                            for (int B = 0; B < 16; ++B) {
                                                const uint32_t f =
                                                    lut[(by[B >> 2] >> (8 * (B & 3))) & 0xffu];
                                                const int pos = 10 * B;
                                                wd[pos >> 5] |= f << (pos & 31);
                                                if ((pos & 31) > 22)
                                                    wd[(pos >> 5) + 1] |= f >> (32 - (pos & 31));
                                            }
                                        } else {
                                            wd[0] = w4.x; wd[1] = w4.y; wd[2] = w4.z; wd[3] = w4.w;
                                        }
                                        if constexpr (S::PERSIST) {
#pragma unroll
                                            for (int jw = 0; jw < NW; ++jw) {
                                                acc[mat][bi][0] = dp4a_us(wd[jw] & 0x03030303u, X[xs][0][4 * jw], acc[mat][bi][0]);
                                                acc[mat][bi][1] = dp4a_us(wd[jw] & 0x0C0C0C0Cu, X[xs][0][4 * jw + 1], acc[mat][bi][1]);
                                                acc[mat][bi][2] = dp4a_us(wd[jw] & 0x30303030u, X[xs][0][4 * jw + 2], acc[mat][bi][2]);
                                                acc[mat][bi][3] = dp4a_us(wd[jw] & 0xC0C0C0C0u, X[xs][0][4 * jw + 3], acc[mat][bi][3]);
                                            }
                                        } else {
                                            uint32_t pl[4 * NW];
#pragma unroll
                                            for (int jw = 0; jw < NW; ++jw) {
                                                pl[4 * jw] = wd[jw] & 0x03030303u;
                                                pl[4 * jw + 1] = wd[jw] & 0x0C0C0C0Cu;
                                                pl[4 * jw + 2] = wd[jw] & 0x30303030u;
                                                pl[4 * jw + 3] = wd[jw] & 0xC0C0C0C0u;
                                            }
#pragma unroll
                                            for (int mq = 0; mq < TQ; ++mq) {
                                                int a0 = 0, a1 = 0, a2 = 0, a3 = 0;
#pragma unroll
                                                for (int jw = 0; jw < NW; ++jw) {
                                                    a0 = dp4a_us(pl[4 * jw], X[xs][mq][4 * jw], a0);
                                                    a1 = dp4a_us(pl[4 * jw + 1], X[xs][mq][4 * jw + 1], a1);
                                                    a2 = dp4a_us(pl[4 * jw + 2], X[xs][mq][4 * jw + 2], a2);
                                                    a3 = dp4a_us(pl[4 * jw + 3], X[xs][mq][4 * jw + 3], a3);
                                                }
                                                acc[mat][bi][m0 + mq] += a0 + (a1 >> 2) + (a2 >> 4) + (a3 >> 6);
                                            }
                                        }
                                    }
                                }
                            }
                        }
                    }
                }
                __syncwarp();
                if (lane == 0)
                    mbar_arrive(empty(slot));
            }
            if (++slot == slots) {
                slot = 0;
                phase ^= 1u;
            }
        }

        // ---- chunk epilogue: fold the k-halves, then the warps (in shared
        // memory); acc = sum c*x~ - sum x~, rescale, bf16
#pragma unroll
        for (int mat = 0; mat < NMAT; ++mat) {
#pragma unroll
            for (int bi = 0; bi < QB; ++bi) {
                if (bi >= qb)
                    break;
#pragma unroll
                for (int m = 0; m < MT; ++m) {
                    int v;
                    if constexpr (S::PERSIST)
                        v = acc[mat][bi][0] + (acc[mat][bi][1] >> 2) + (acc[mat][bi][2] >> 4) +
                            (acc[mat][bi][3] >> 6);
                    else
                        v = acc[mat][bi][m];
                    v += __shfl_xor_sync(0xffffffffu, v, 1);
                    if (t == 0)
                        red[mat * red_stride + (warp * p.red_blocks * 16 + bi * 16 + r) * MT + m] = v;
                }
            }
        }
        compute_sync();
        if (!*abort_flag) {
            const int rows = qb * 16;
            for (int o = ctid; o < rows * M; o += CTHREADS) {
                const int m = o / rows;
                const int rl = o - m * rows;
                const int n = (blk0 + b0) * 16 + rl;
                if (n < N) {
                    // row sum of matrix `mat` minus the sum of the x~ it read
                    auto row_acc = [&](int mat) {
                        const int xs = mat < NX ? mat : NX - 1;
                        int a = 0, s = 0;
#pragma unroll
                        for (int w = 0; w < CWARPS; ++w) {
                            a += red[mat * red_stride + (w * p.red_blocks * 16 + rl) * MT + m];
                            s += red_s(xs)[m * CWARPS + w];
                        }
                        return a - s;
                    };
                    const size_t oi = static_cast<size_t>(m) * N + n;
                    const int a = row_acc(0);
                    const uint16_t y0 = rescale_bf16(a, out_scale(beta_sm(0)[m], P.gamma));
                    if constexpr (FFN) {
                        const uint16_t y1 =
                            rescale_bf16(row_acc(1), out_scale(beta_sm(NX - 1)[m], P.gamma2));
                        if (P.y != nullptr)
                            P.y[oi] = y0;
                        if (P.y2 != nullptr)
                            P.y2[oi] = y1;
                        // h = (r * r) * up with r = max(gate, 0), fp32 (exact
                        // for bf16 operands)
                        const float gv = __uint_as_float(static_cast<uint32_t>(y0) << 16);
                        const float uv = __uint_as_float(static_cast<uint32_t>(y1) << 16);
                        const float rg = gv > 0.0f ? gv : 0.0f;
                        P.h[oi] = __fmul_rn(__fmul_rn(rg, rg), uv);
                    } else {
                        P.y[oi] = y0;
                    }
                    if (P.acc_dbg != nullptr)
                        P.acc_dbg[oi] = a;
                }
            }
        }
        // the reduction area is reused by the next chunk
        compute_sync();
    }
}

}  // namespace gemv
}  // namespace bitlinear
