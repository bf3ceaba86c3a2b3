// Device helpers shared by the BitLinear kernels: inline PTX for mbarriers,
// bulk / tensor TMA copies, tcgen05 (TMEM, UMMA) and programmatic dependent
// launch, plus bounded waits that record a fault instead of hanging.
#pragma once

#include <cuda.h>
#include <cuda_bf16.h>
#include <cuda_runtime.h>
#include <stdint.h>

namespace bitlinear {

// Device-side fault word (read and cleared by bitlinear_get_fault).
__device__ unsigned int g_fault_word;

enum FaultCode : unsigned int {
    FAULT_NONE = 0,
    FAULT_WAIT_TIMEOUT = 1,
};

// ------------------------------------------------------------------ basics

__device__ __forceinline__ uint32_t smem_u32(const void *p)
{
    return static_cast<uint32_t>(__cvta_generic_to_shared(p));
}

__device__ __forceinline__ uint64_t global_timer_ns()
{
    uint64_t t;
    asm volatile("mov.u64 %0, %%globaltimer;" : "=l"(t));
    return t;
}

// dp4a on signed bytes: sum_i a_i * b_i + c.
__device__ __forceinline__ int dp4a_ss(uint32_t a, uint32_t b, int c)
{
    return __dp4a(static_cast<int>(a), static_cast<int>(b), c);
}

// ---------------------------------------------------------------- mbarrier

__device__ __forceinline__ void mbar_init(uint32_t bar, uint32_t count)
{
    asm volatile("mbarrier.init.shared::cta.b64 [%0], %1;" ::"r"(bar), "r"(count));
}

__device__ __forceinline__ void fence_barrier_init()
{
    asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
}

__device__ __forceinline__ void mbar_arrive(uint32_t bar)
{
    asm volatile("mbarrier.arrive.shared::cta.b64 _, [%0];" ::"r"(bar) : "memory");
}

__device__ __forceinline__ void mbar_arrive_expect_tx(uint32_t bar, uint32_t bytes)
{
    asm volatile("mbarrier.arrive.expect_tx.shared::cta.b64 _, [%0], %1;" ::"r"(bar),
                 "r"(bytes)
                 : "memory");
}

__device__ __forceinline__ bool mbar_try_wait(uint32_t bar, uint32_t parity)
{
    uint32_t done;
    asm volatile(
        "{\n\t.reg .pred p;\n\t"
        "mbarrier.try_wait.parity.shared::cta.b64 p, [%1], %2;\n\t"
        "selp.u32 %0, 1, 0, p;\n\t}"
        : "=r"(done)
        : "r"(bar), "r"(parity)
        : "memory");
    return done != 0;
}

// Wait until the phase with the given parity of the barrier has completed.
// Gives up after limit_ns nanoseconds, or as soon as *abort becomes nonzero:
// on a timeout it records FAULT_WAIT_TIMEOUT, raises *abort so that the other
// roles of the block stop waiting too, and returns false.
__device__ __forceinline__ bool mbar_wait_bounded(uint32_t bar, uint32_t parity,
                                                  volatile int *abort,
                                                  uint64_t limit_ns)
{
    if (mbar_try_wait(bar, parity))
        return true;
    const uint64_t t0 = global_timer_ns();
    for (uint32_t spin = 1;; ++spin) {
        if (mbar_try_wait(bar, parity))
            return true;
        if ((spin & 63u) == 0u) {
            if (*abort)
                return false;
            if (global_timer_ns() - t0 > limit_ns) {
                atomicOr(&g_fault_word, FAULT_WAIT_TIMEOUT);
                *abort = 1;
                return false;
            }
        }
    }
}

// mbarrier.try_wait with a suspend-time hint: a thread whose phase has not
// completed sleeps until it does or about hint_ns nanoseconds pass, instead of
// spinning (the waiting warps then take no issue slots from working ones).
__device__ __forceinline__ bool mbar_try_wait_sleep(uint32_t bar, uint32_t parity,
                                                    uint32_t hint_ns)
{
    uint32_t done;
    asm volatile(
        "{\n\t.reg .pred p;\n\t"
        "mbarrier.try_wait.parity.shared::cta.b64 p, [%1], %2, %3;\n\t"
        "selp.u32 %0, 1, 0, p;\n\t}"
        : "=r"(done)
        : "r"(bar), "r"(parity), "r"(hint_ns)
        : "memory");
    return done != 0;
}

// mbar_wait_bounded for long waits (data from HBM): each try sleeps up to
// 20 us, and the limit and the abort flag are checked after every try.
__device__ __forceinline__ bool mbar_wait_sleep_bounded(uint32_t bar, uint32_t parity,
                                                        volatile int *abort, uint64_t limit_ns)
{
    if (mbar_try_wait_sleep(bar, parity, 20000u))
        return true;
    const uint64_t t0 = global_timer_ns();
    for (;;) {
        if (mbar_try_wait_sleep(bar, parity, 20000u))
            return true;
        if (*abort)
            return false;
        if (global_timer_ns() - t0 > limit_ns) {
            atomicOr(&g_fault_word, FAULT_WAIT_TIMEOUT);
            *abort = 1;
            return false;
        }
    }
}

// Lane 0 waits (sleeping between tries), the verdict is broadcast, and the
// warp re-converges.
__device__ __forceinline__ bool warp_wait_sleep_bounded(uint32_t bar, uint32_t parity,
                                                        volatile int *abort, uint64_t limit_ns)
{
    int ok = 0;
    if ((threadIdx.x & 31) == 0)
        ok = mbar_wait_sleep_bounded(bar, parity, abort, limit_ns) ? 1 : 0;
    ok = __shfl_sync(0xffffffffu, ok, 0);
    __syncwarp();
    return ok != 0;
}

// Lane 0 waits, the verdict is broadcast, and the warp re-converges.
__device__ __forceinline__ bool warp_wait_bounded(uint32_t bar, uint32_t parity,
                                                  volatile int *abort, uint64_t limit_ns)
{
    int ok = 0;
    if ((threadIdx.x & 31) == 0)
        ok = mbar_wait_bounded(bar, parity, abort, limit_ns) ? 1 : 0;
    ok = __shfl_sync(0xffffffffu, ok, 0);
    __syncwarp();
    return ok != 0;
}

__device__ __forceinline__ bool mbar_test_wait(uint32_t bar, uint32_t parity)
{
    uint32_t done;
    asm volatile(
        "{\n\t.reg .pred p;\n\t"
        "mbarrier.test_wait.parity.shared::cta.b64 p, [%1], %2;\n\t"
        "selp.u32 %0, 1, 0, p;\n\t}"
        : "=r"(done)
        : "r"(bar), "r"(parity)
        : "memory");
    return done != 0;
}

// Waits for the given phases of two barriers at once: every lane of the warp
// polls both (non-blocking tests), and the warp leaves together when all
// lanes have seen both complete, so the two waits overlap instead of running
// one after the other. Bounded like mbar_wait_bounded (lane 0 keeps the time
// and the abort flag; the verdict is shared).
__device__ __forceinline__ bool warp_wait2_bounded(uint32_t bar1, uint32_t parity1, uint32_t bar2,
                                                   uint32_t parity2, volatile int *abort,
                                                   uint64_t limit_ns)
{
    bool d1 = false, d2 = false;
    uint64_t t0 = 0;
    for (uint32_t spin = 0;; ++spin) {
        d1 = d1 || mbar_test_wait(bar1, parity1);
        d2 = d2 || mbar_test_wait(bar2, parity2);
        if (__all_sync(0xffffffffu, d1 && d2))
            return true;
        if ((spin & 63u) == 0u) {
            int stop = 0;
            if ((threadIdx.x & 31) == 0) {
                if (spin == 0) {
                    t0 = global_timer_ns();
                } else if (*abort) {
                    stop = 1;
                } else if (global_timer_ns() - t0 > limit_ns) {
                    atomicOr(&g_fault_word, FAULT_WAIT_TIMEOUT);
                    *abort = 1;
                    stop = 1;
                }
            }
            if (__shfl_sync(0xffffffffu, stop, 0))
                return false;
        }
    }
}

// Bounded wait that ignores the abort flag: used only to drain this thread's
// own asynchronous work (copies, MMAs) before the block exits.
__device__ __forceinline__ void drain_wait(uint32_t bar, uint32_t parity, uint64_t limit_ns)
{
    const uint64_t t0 = global_timer_ns();
    while (!mbar_try_wait(bar, parity)) {
        if (global_timer_ns() - t0 > limit_ns) {
            atomicOr(&g_fault_word, FAULT_WAIT_TIMEOUT);
            return;
        }
    }
}

// -------------------------------------------------------------- bulk / TMA

// Non-tensor bulk copy global -> shared, completion counted on an mbarrier.
// dst, src 16-byte aligned, bytes a multiple of 16.
__device__ __forceinline__ void bulk_g2s(uint32_t dst, const void *src, uint32_t bytes,
                                         uint32_t bar)
{
    asm volatile(
        "cp.async.bulk.shared::cluster.global.mbarrier::complete_tx::bytes [%0], [%1], %2, [%3];" ::"r"(
            dst),
        "l"(src), "r"(bytes), "r"(bar)
        : "memory");
}

// 16-byte asynchronous copy global -> shared (L2 only); dst and src 16-byte
// aligned. Complete for the issuing thread after cp_async_wait_all.
__device__ __forceinline__ void cp_async16(uint32_t dst, const void *src)
{
    asm volatile("cp.async.cg.shared.global [%0], [%1], 16;" ::"r"(dst), "l"(src) : "memory");
}

__device__ __forceinline__ void cp_async_wait_all()
{
    asm volatile("cp.async.wait_all;" ::: "memory");
}

// 3-D tiled tensor copy global -> this CTA's shared memory.
__device__ __forceinline__ void tma_load_3d(uint32_t dst, const CUtensorMap *map, int c0, int c1,
                                            int c2, uint32_t bar)
{
    asm volatile(
        "cp.async.bulk.tensor.3d.shared::cluster.global.mbarrier::complete_tx::bytes "
        "[%0], [%1, {%2, %3, %4}], [%5];" ::"r"(dst),
        "l"(reinterpret_cast<uint64_t>(map)), "r"(c0), "r"(c1), "r"(c2), "r"(bar)
        : "memory");
}

__device__ __forceinline__ void prefetch_tensormap(const CUtensorMap *map)
{
    asm volatile("prefetch.tensormap [%0];" ::"l"(reinterpret_cast<uint64_t>(map))
                 : "memory");
}

// ----------------------------------------------------------------- tcgen05

__device__ __forceinline__ void tmem_alloc(uint32_t dst_smem, uint32_t cols)
{
    asm volatile("tcgen05.alloc.cta_group::1.sync.aligned.shared::cta.b32 [%0], %1;" ::"r"(
                     dst_smem),
                 "r"(cols)
                 : "memory");
}

__device__ __forceinline__ void tmem_relinquish()
{
    asm volatile("tcgen05.relinquish_alloc_permit.cta_group::1.sync.aligned;" ::: "memory");
}

__device__ __forceinline__ void tmem_dealloc(uint32_t taddr, uint32_t cols)
{
    asm volatile("tcgen05.dealloc.cta_group::1.sync.aligned.b32 %0, %1;" ::"r"(taddr),
                 "r"(cols)
                 : "memory");
}

__device__ __forceinline__ void tc_fence_before_sync()
{
    asm volatile("tcgen05.fence::before_thread_sync;" ::: "memory");
}

__device__ __forceinline__ void tc_fence_after_sync()
{
    asm volatile("tcgen05.fence::after_thread_sync;" ::: "memory");
}

// D[tmem] (+)= A[tmem] * B[smem]^T, int8 inputs, int32 accumulator. For
// M = 128 the A tile occupies TMEM lanes 0..127 (lane = row) and k runs along
// the columns, four int8 values per 32-bit column (k = 4c .. 4c+3 in bytes
// 0..3), eight columns per k-step of 32. The B descriptor comes as its two
// 32-bit words, so that an issuing loop can step the start address (the low
// word's bits 0-13, in 16-byte units) with one 32-bit add per MMA.
__device__ __forceinline__ void umma_i8_tmem_a_w(uint32_t d_tmem, uint32_t a_tmem, uint32_t b_lo,
                                                 uint32_t b_hi, uint32_t idesc,
                                                 uint32_t accumulate)
{
    asm volatile(
        "{\n\t.reg .pred p;\n\t.reg .b64 bd;\n\t"
        "setp.ne.b32 p, %5, 0;\n\t"
        "mov.b64 bd, {%2, %3};\n\t"
        "tcgen05.mma.cta_group::1.kind::i8 [%0], [%1], bd, %4, p;\n\t}" ::"r"(d_tmem),
        "r"(a_tmem), "r"(b_lo), "r"(b_hi), "r"(idesc), "r"(accumulate)
        : "memory");
}

// Arrive (once) on an mbarrier when all previously issued tcgen05.mma of
// this thread have completed.
__device__ __forceinline__ void umma_commit(uint32_t bar)
{
    asm volatile(
        "tcgen05.commit.cta_group::1.mbarrier::arrive::one.shared::cluster.b64 [%0];" ::"r"(bar)
        : "memory");
}

// 32 lanes x 32 consecutive 32-bit TMEM columns -> 32 registers per thread.
__device__ __forceinline__ void tmem_ld_32x32b_x32(uint32_t taddr, uint32_t (&r)[32])
{
    asm volatile(
        "tcgen05.ld.sync.aligned.32x32b.x32.b32 "
        "{%0, %1, %2, %3, %4, %5, %6, %7, %8, %9, %10, %11, %12, %13, %14, %15, "
        "%16, %17, %18, %19, %20, %21, %22, %23, %24, %25, %26, %27, %28, %29, %30, %31}, "
        "[%32];"
        : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3]), "=r"(r[4]), "=r"(r[5]), "=r"(r[6]),
          "=r"(r[7]), "=r"(r[8]), "=r"(r[9]), "=r"(r[10]), "=r"(r[11]), "=r"(r[12]),
          "=r"(r[13]), "=r"(r[14]), "=r"(r[15]), "=r"(r[16]), "=r"(r[17]), "=r"(r[18]),
          "=r"(r[19]), "=r"(r[20]), "=r"(r[21]), "=r"(r[22]), "=r"(r[23]), "=r"(r[24]),
          "=r"(r[25]), "=r"(r[26]), "=r"(r[27]), "=r"(r[28]), "=r"(r[29]), "=r"(r[30]),
          "=r"(r[31])
        : "r"(taddr)
        : "memory");
}

// 32 registers per thread -> 32 lanes x 32 consecutive 32-bit TMEM columns.
__device__ __forceinline__ void tmem_st_32x32b_x32(uint32_t taddr, const uint32_t (&r)[32])
{
    asm volatile(
        "tcgen05.st.sync.aligned.32x32b.x32.b32 [%0], "
        "{%1, %2, %3, %4, %5, %6, %7, %8, %9, %10, %11, %12, %13, %14, %15, %16, "
        "%17, %18, %19, %20, %21, %22, %23, %24, %25, %26, %27, %28, %29, %30, %31, %32};"
        ::"r"(taddr), "r"(r[0]), "r"(r[1]), "r"(r[2]), "r"(r[3]), "r"(r[4]), "r"(r[5]),
        "r"(r[6]), "r"(r[7]), "r"(r[8]), "r"(r[9]), "r"(r[10]), "r"(r[11]), "r"(r[12]),
        "r"(r[13]), "r"(r[14]), "r"(r[15]), "r"(r[16]), "r"(r[17]), "r"(r[18]), "r"(r[19]),
        "r"(r[20]), "r"(r[21]), "r"(r[22]), "r"(r[23]), "r"(r[24]), "r"(r[25]), "r"(r[26]),
        "r"(r[27]), "r"(r[28]), "r"(r[29]), "r"(r[30]), "r"(r[31])
        : "memory");
}

__device__ __forceinline__ void tmem_st_wait()
{
    asm volatile("tcgen05.wait::st.sync.aligned;" ::: "memory");
}

__device__ __forceinline__ void tmem_ld_wait()
{
    asm volatile("tcgen05.wait::ld.sync.aligned;" ::: "memory");
}

// Shared-memory matrix descriptor for a K-major operand tile stored in the
// 128-byte swizzled layout: rows of 128 bytes, 8-row atoms of 1024 bytes
// (stride-dimension byte offset), 16-byte chunks XOR-ed with (row % 8).
__device__ __forceinline__ uint64_t smem_desc_k128_sw128(uint32_t saddr)
{
    uint64_t d = 0;
    d |= static_cast<uint64_t>((saddr & 0x3FFFFu) >> 4);  // start address
    d |= static_cast<uint64_t>(1) << 16;                   // leading byte offset (unused)
    d |= static_cast<uint64_t>(1024 >> 4) << 32;           // stride byte offset
    d |= static_cast<uint64_t>(1) << 46;                   // descriptor version (sm_100)
    d |= static_cast<uint64_t>(2) << 61;                   // 128-byte swizzle
    return d;
}

// Instruction descriptor: kind::i8, s8 x s8 -> s32, both operands K-major.
__host__ __device__ constexpr uint32_t idesc_i8_s32(int m, int n)
{
    return (2u << 4)                                  // D format: s32
           | (1u << 7)                                // A format: signed 8-bit
           | (1u << 10)                               // B format: signed 8-bit
           | (static_cast<uint32_t>(n >> 3) << 17)    // N / 8
           | (static_cast<uint32_t>(m >> 4) << 24);   // M / 16
}

// AND of v over the `nthreads` threads (whole warps) that use named barrier
// `id`; every one of them must call it. Lets a group of warps take a bounded
// wait's verdict together, so that none of them is left at a later barrier.
__device__ __forceinline__ bool named_bar_and(int id, int nthreads, bool v)
{
    uint32_t r;
    asm volatile(
        "{\n\t.reg .pred p, q;\n\t"
        "setp.ne.u32 p, %1, 0;\n\t"
        "bar.red.and.pred q, %2, %3, p;\n\t"
        "selp.u32 %0, 1, 0, q;\n\t}"
        : "=r"(r)
        : "r"(static_cast<uint32_t>(v)), "r"(id), "r"(nthreads)
        : "memory");
    return r != 0;
}

// ------------------------------------------------ inter-block flags (L2)

__device__ __forceinline__ int ld_acquire_gpu(const int *p)
{
    int v;
    asm volatile("ld.acquire.gpu.global.b32 %0, [%1];" : "=r"(v) : "l"(p) : "memory");
    return v;
}

__device__ __forceinline__ void st_release_gpu(int *p, int v)
{
    asm volatile("st.release.gpu.global.b32 [%0], %1;" ::"l"(p), "r"(v) : "memory");
}

// --------------------------------------------- programmatic dependent launch

// Wait until the grids this one depends on have completed and their memory
// is visible (no-op when launched without the programmatic attribute).
__device__ __forceinline__ void pdl_wait()
{
    asm volatile("griddepcontrol.wait;" ::: "memory");
}

// Allow the next grid in the stream to begin launching.
__device__ __forceinline__ void pdl_launch_dependents()
{
    asm volatile("griddepcontrol.launch_dependents;" ::: "memory");
}

// ------------------------------------------------------ quantisation helpers

// Loads 8 consecutive activations starting at element e of a row as fp32
// (bf16 widening is exact).
template <bool BF16>
__device__ __forceinline__ void load8(const void *row, int e, float (&v)[8])
{
    if constexpr (BF16) {
        const uint4 raw = __ldg(reinterpret_cast<const uint4 *>(
            static_cast<const __nv_bfloat16 *>(row) + e));
        const uint32_t w[4] = {raw.x, raw.y, raw.z, raw.w};
#pragma unroll
        for (int i = 0; i < 4; ++i) {
            v[2 * i] = __uint_as_float(w[i] << 16);
            v[2 * i + 1] = __uint_as_float(w[i] & 0xffff0000u);
        }
    } else {
        const float4 a = __ldg(reinterpret_cast<const float4 *>(static_cast<const float *>(row) + e));
        const float4 b =
            __ldg(reinterpret_cast<const float4 *>(static_cast<const float *>(row) + e + 4));
        v[0] = a.x; v[1] = a.y; v[2] = a.z; v[3] = a.w;
        v[4] = b.x; v[5] = b.y; v[6] = b.z; v[7] = b.w;
    }
}

// Raw 8-activation vectors: four bf16 pairs or eight fp32 words.
template <bool BF16>
struct Vec8 {
    static constexpr int WORDS = BF16 ? 4 : 8;
    uint32_t w[WORDS];

    __device__ __forceinline__ void load(const void *row, int e)
    {
        const uint4 *src = reinterpret_cast<const uint4 *>(static_cast<const char *>(row) +
                                                           static_cast<size_t>(e) * (BF16 ? 2 : 4));
#pragma unroll
        for (int i = 0; i < WORDS / 4; ++i) {
            const uint4 v = __ldg(src + i);
            w[4 * i] = v.x; w[4 * i + 1] = v.y; w[4 * i + 2] = v.z; w[4 * i + 3] = v.w;
        }
    }

    __device__ __forceinline__ float get(int i) const
    {
        if constexpr (BF16)
            return __uint_as_float((i & 1) ? (w[i >> 1] & 0xffff0000u) : (w[i >> 1] << 16));
        else
            return __uint_as_float(w[i]);
    }
};

// RMS normalisation of one activation: (x * r) * g, two correctly rounded
// fp32 products in the order torch's RMSNorm applies them (r = 1 / sqrt(mean
// x^2 + eps) of the token, g the channel's gain).
__device__ __forceinline__ float norm1(float x, float r, float g)
{
    return __fmul_rn(__fmul_rn(x, r), g);
}

// r = 1 / sqrt(ss / K + eps) from a token's sum of squares in double: the
// mean rounded once to fp32, then IEEE fp32 add, square root and division.
__device__ __forceinline__ float rms_scale(double ss, int K, float eps)
{
    const float ms = __double2float_rn(__ddiv_rn(ss, static_cast<double>(K)));
    return __fdiv_rn(1.0f, __fsqrt_rn(__fadd_rn(ms, eps)));
}

// Sum of a double over the warp (xor butterfly: every lane ends with the
// same bits, as each step adds two commuted copies of the same partial sums).
__device__ __forceinline__ double warp_sum_f64(double v)
{
#pragma unroll
    for (int o = 16; o > 0; o >>= 1)
        v = __dadd_rn(v, __shfl_xor_sync(0xffffffffu, v, o));
    return v;
}

// rint(v) for |v| < 2^22, as the bit pattern of an fp32 sum: adding 1.5 * 2^23
// puts v + c in [2^23, 2^24), where the spacing is 1, so the IEEE addition
// rounds v to an integer (ties to even, as rint) and the result's bits are
// 0x4B400000 + rint(v). Its low byte is rint(v) as a two's-complement byte. A
// full-rate addition in place of a float-to-integer conversion.
__device__ __forceinline__ uint32_t rint_bits(float v)
{
    return __float_as_uint(__fadd_rn(v, 12582912.0f));
}

// x~ = clamp(round_half_even(x * scale), -128, 127): the product rounded to
// fp32 first, as the listing computes it, then to an integer. With scale =
// 127 / beta and beta the absmax of the row (or 1e-5 above every |x|),
// |x * scale| <= 127, so the clamp never binds; it is kept here for callers
// whose scale is not that.
// Lane-wise unsigned maximum of two pairs of 16-bit fields.
__device__ __forceinline__ uint32_t max_u16x2(uint32_t a, uint32_t b)
{
    uint32_t d;
    asm("max.u16x2 %0, %1, %2;" : "=r"(d) : "r"(a), "r"(b));
    return d;
}

__device__ __forceinline__ int quant1(float x, float scale)
{
    const int q = static_cast<int>(rint_bits(__fmul_rn(x, scale)) - 0x4B400000u);
    return min(127, max(-128, q));
}

// (beta * gamma) / 127 in fp32, the order of the listing's rescale.
__device__ __forceinline__ float out_scale(float beta, float gamma)
{
    return __fdiv_rn(__fmul_rn(beta, gamma), 127.0f);
}

__device__ __forceinline__ uint16_t rescale_bf16(int acc, float s)
{
    const float v = __fmul_rn(__int2float_rn(acc), s);
    return __bfloat16_as_ushort(__float2bfloat16_rn(v));
}

}  // namespace bitlinear
