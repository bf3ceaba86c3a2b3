// C ABI of libbitlinear (declared in include/bitlinear.h): argument checks,
// kernel choice and launches of the BitLinear W1.58A8 matmul on sm_100a.
//
// All kernels live in this translation unit so that they share the device
// fault word; the offline packer is host code in pack.cpp.

#include <cuda.h>
#include <cuda_runtime.h>

#include <algorithm>
#include <atomic>
#include <cfloat>
#include <climits>
#include <cstdint>
#include <cstdlib>
#include <cstring>
#include <mutex>
#include <utility>

#include "../../include/bitlinear.h"
#include "common.cuh"
#include "gemm_ws.cuh"
#include "gemv.cuh"
#include "quant_act.cuh"
#include "stage_io.cuh"
#include "ffn_act.cuh"

using namespace bitlinear;

namespace {

constexpr int64_t kMaxK = 65536;
constexpr int kGemvMaxM = 16;
constexpr int64_t kGemvMaxXqBytes = 196608;       // at most M * K bytes of x~ in shared memory
constexpr int kSmemOptinSm100 = 227 * 1024;        // opt-in shared memory per block on sm_100
constexpr int64_t kAutoGemvMaxM = 6;                // above: tensor-core path
// Split the k-range of fewer tiles than CTAs only when a CTA saves more than
// this many 256-k blocks (each about half a microsecond) by it.
constexpr double kSplitMinSavedBlocks = 10.0;
// A split launch with fewer tiles than CTAs gives each CTA at least this many
// k-blocks of 256: a tile shared by many CTAs pays one partial-sum hand-off
// per contributor.
constexpr int64_t kSplitMinCtaBlocks = 8;
// k-blocks of 256 per CTA from which the small token tiles take 512-k stages
constexpr int64_t kDeepStageMinBlocks = 8;
constexpr uint64_t kWaitLimitNs = 1000000000ull;  // 1 s: far above any legitimate wait
constexpr int kMaxDevices = 64;

bool aligned(const void *p, uintptr_t a) { return (reinterpret_cast<uintptr_t>(p) % a) == 0; }

// Token tile of a GEMV launch for up to M tokens.
int gemv_tile(int64_t M) { return M <= 1 ? 1 : M <= 2 ? 2 : M <= 4 ? 4 : M <= 8 ? 8 : 16; }

// Largest x~ (M * K bytes; for a group, the largest problem's) a GEMV launch
// for up to M tokens admits. With the smallest stage geometry (one row block
// of 8 k-groups per slot, two slots) the launch then still fits in sm_100's
// opt-in shared memory beside the reduction area and the normalising form's
// arrays, for every token tile.
int64_t gemv_max_xq(int64_t M)
{
    const int MT = gemv_tile(M);
    return std::min<int64_t>(
        kGemvMaxXqBytes,
        kSmemOptinSm100 - gemv::smem_bytes(MT, 0, 2, 8 * gemv::PIECE, 1, true));
}

bool gemv_fits(int64_t M, int64_t K) { return M <= kGemvMaxM && M * K <= gemv_max_xq(M); }

size_t round_up(size_t v, size_t a) { return (v + a - 1) / a * a; }

struct DeviceInfo {
    int id = 0;
    int sms = 0;
    int max_smem_optin = 0;
};

DeviceInfo g_devices[kMaxDevices];
std::once_flag g_device_once[kMaxDevices];

int current_device(DeviceInfo **info)
{
    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= kMaxDevices)
        return BITLINEAR_ERR_CUDA;
    std::call_once(g_device_once[dev], [dev] {
        g_devices[dev].id = dev;
        cudaDeviceGetAttribute(&g_devices[dev].sms, cudaDevAttrMultiProcessorCount, dev);
        cudaDeviceGetAttribute(&g_devices[dev].max_smem_optin,
                               cudaDevAttrMaxSharedMemoryPerBlockOptin, dev);
    });
    *info = &g_devices[dev];
    return g_devices[dev].sms > 0 ? BITLINEAR_OK : BITLINEAR_ERR_CUDA;
}

// Opt a kernel into more than 48 KiB of dynamic shared memory. The attribute
// is per function and device; it is set once (and raised when a larger size
// is needed) so that launches inside a stream capture make no such call.
template <auto Kernel>
cudaError_t allow_smem(int dev, int bytes)
{
    static std::atomic<int> granted[kMaxDevices];
    if (bytes <= 48 * 1024 || granted[dev].load(std::memory_order_acquire) >= bytes)
        return cudaSuccess;
    cudaError_t e =
        cudaFuncSetAttribute(Kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, bytes);
    if (e == cudaSuccess) {
        int cur = granted[dev].load();
        while (cur < bytes && !granted[dev].compare_exchange_weak(cur, bytes)) {
        }
    }
    return e;
}

// ------------------------------------------------------------ tensor maps

using EncodeTiledFn = CUresult (*)(CUtensorMap *, CUtensorMapDataType, cuuint32_t, void *,
                                   const cuuint64_t *, const cuuint64_t *, const cuuint32_t *,
                                   const cuuint32_t *, CUtensorMapInterleave, CUtensorMapSwizzle,
                                   CUtensorMapL2promotion, CUtensorMapFloatOOBfill);

EncodeTiledFn encode_fn()
{
    static EncodeTiledFn fn = [] {
        void *p = nullptr;
        cudaDriverEntryPointQueryResult q;
        if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &p, cudaEnableDefault, &q) !=
                cudaSuccess ||
            q != cudaDriverEntryPointSuccess)
            return static_cast<EncodeTiledFn>(nullptr);
        return reinterpret_cast<EncodeTiledFn>(p);
    }();
    return fn;
}

// Programmatic dependent launch: a kernel launched this way may start while
// the previous kernel in the stream is still running; it reads nothing the
// previous work may have written (activations, workspace) before its
// griddepcontrol.wait, except the packed weights, which the GEMV starts
// streaming at once. On by default; BITLINEAR_PDL=0 in the environment turns
// it off (every launch then waits for the previous one as usual).
bool pdl_enabled()
{
    static const bool on = [] {
        const char *v = std::getenv("BITLINEAR_PDL");
        return !(v != nullptr && v[0] == '0');
    }();
    return on;
}

template <typename... KArgs, typename... Args>
cudaError_t launch(void (*kernel)(KArgs...), dim3 grid, dim3 block, size_t smem,
                   cudaStream_t st, Args &&...args)
{
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = grid;
    cfg.blockDim = block;
    cfg.dynamicSmemBytes = smem;
    cfg.stream = st;
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    attr[0].val.programmaticStreamSerializationAllowed = 1;
    cfg.attrs = attr;
    cfg.numAttrs = pdl_enabled() ? 1 : 0;
    return cudaLaunchKernelEx(&cfg, kernel, std::forward<Args>(args)...);
}

// x~ [M][K] int8 as a 3-D tensor {128 B, M rows, K/128 chunks} (strides K
// and 128 bytes), boxed as {128, box_rows, groups} with the 128-byte swizzle:
// one box is a (128 groups)-k slice of box_rows tokens, landing in shared
// memory as `groups` swizzled [box_rows][128] sub-tiles.
bool make_map_xq(CUtensorMap *map, const void *ptr, int64_t M, int64_t K, uint32_t box_rows,
                 uint32_t groups)
{
    EncodeTiledFn fn = encode_fn();
    if (fn == nullptr)
        return false;
    const cuuint64_t dims[3] = {128, static_cast<cuuint64_t>(M), static_cast<cuuint64_t>(K / 128)};
    const cuuint64_t strides[2] = {static_cast<cuuint64_t>(K), 128};
    const cuuint32_t box[3] = {128, box_rows, groups};
    const cuuint32_t estride[3] = {1, 1, 1};
    CUresult r = fn(map, CU_TENSOR_MAP_DATA_TYPE_UINT8, 3, const_cast<void *>(ptr), dims, strides,
                    box, estride, CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
                    CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
    return r == CUDA_SUCCESS;
}

// The packed weights as a 3-D tensor of 8-byte elements {64 (= the 512 bytes
// of one row block and 128-k group), K/128 groups, ceil(N/16) row blocks}
// (strides 512 and 16 * K/4 bytes), boxed as {64, groups, box_rows/16}: one
// box is box_rows rows x (128 groups) weights, landing as
// [box_rows/16][groups][16 rows][32 B].
bool make_map_packed(CUtensorMap *map, const void *ptr, int64_t N, int64_t K, uint32_t box_rows,
                     uint32_t groups)
{
    EncodeTiledFn fn = encode_fn();
    if (fn == nullptr)
        return false;
    const cuuint64_t dims[3] = {64, static_cast<cuuint64_t>(K / 128),
                                static_cast<cuuint64_t>((N + 15) / 16)};
    const cuuint64_t strides[2] = {512, static_cast<cuuint64_t>(16 * (K / 4))};
    const cuuint32_t box[3] = {64, groups, box_rows / 16};
    const cuuint32_t estride[3] = {1, 1, 1};
    CUresult r = fn(map, CU_TENSOR_MAP_DATA_TYPE_UINT64, 3, const_cast<void *>(ptr), dims, strides,
                    box, estride, CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_NONE,
                    CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
    return r == CUDA_SUCCESS;
}

int launch_status(cudaError_t e)
{
    if (e != cudaSuccess) {
        cudaGetLastError();
        return BITLINEAR_ERR_CUDA;
    }
    return cudaGetLastError() == cudaSuccess ? BITLINEAR_OK : BITLINEAR_ERR_CUDA;
}

// ----------------------------------------------------------- quantisation

template <bool BF16, int CACHE, int WPR>
cudaError_t launch_qa(const void *x, int M, int K, int8_t *xq, float *beta, int *rowsum,
                      cudaStream_t st, int *clear, int n_clear, const float *gain, float eps)
{
    constexpr int rpb = qa::rows_per_block<WPR>();
    const dim3 grid((M + rpb - 1) / rpb);
    if (gain != nullptr)
        return launch(qa::quant_act_kernel<BF16, CACHE, WPR, true>, grid, dim3(qa::THREADS), 0,
                      st, x, M, K, xq, beta, rowsum, clear, n_clear, gain, eps);
    return launch(qa::quant_act_kernel<BF16, CACHE, WPR, false>, grid, dim3(qa::THREADS), 0, st,
                  x, M, K, xq, beta, rowsum, clear, n_clear, gain, eps);
}

// Prefill batches (at least kStagedQuantMinRows tokens, four or more rows in
// kStagedQuantSmem bytes) take the staged kernel: R rows per block in shared
// memory, one wave for the batch.
constexpr int kStagedQuantMinRows = 1024;
constexpr int kStagedQuantSmem = 112 * 1024;

template <bool BF16, bool NORM>
cudaError_t launch_qa_staged_t(const void *x, int M, int K, int rpb, int8_t *xq, float *beta,
                               int *rowsum, cudaStream_t st, int *clear, int n_clear,
                               const float *gain, float eps, int dev)
{
    const int smem = rpb * K * (BF16 ? 2 : 4);
    cudaError_t e = allow_smem<qa::quant_act_staged_kernel<BF16, NORM>>(dev, smem);
    if (e == cudaSuccess)
        e = launch(qa::quant_act_staged_kernel<BF16, NORM>, dim3((M + rpb - 1) / rpb),
                   dim3(qa::THREADS), smem, st, x, M, K, rpb, xq, beta, rowsum, clear, n_clear,
                   gain, eps, kWaitLimitNs);
    return e;
}

int launch_qa_staged(const void *x, bool bf16, int M, int K, int rpb, int8_t *xq, float *beta,
                     int *rowsum, cudaStream_t st, int *clear, int n_clear, const float *gain,
                     float eps, int dev)
{
    cudaError_t e;
    if (gain != nullptr)
        e = bf16 ? launch_qa_staged_t<true, true>(x, M, K, rpb, xq, beta, rowsum, st, clear,
                                                  n_clear, gain, eps, dev)
                 : launch_qa_staged_t<false, true>(x, M, K, rpb, xq, beta, rowsum, st, clear,
                                                   n_clear, gain, eps, dev);
    else
        e = bf16 ? launch_qa_staged_t<true, false>(x, M, K, rpb, xq, beta, rowsum, st, clear,
                                                   n_clear, gain, eps, dev)
                 : launch_qa_staged_t<false, false>(x, M, K, rpb, xq, beta, rowsum, st, clear,
                                                    n_clear, gain, eps, dev);
    return launch_status(e);
}

// Register cache per lane and warps per row by row length: every lane holds
// its whole share of a row in registers up to 16384 bf16 (8192 fp32)
// elements per row, so a row is read from memory once and small batches are
// not held up by dependent re-reads; longer rows take eight warps and
// re-read the rest. A non-null gain RMS-normalises each row first.
int launch_quant_act(const void *x, bitlinear_dtype xdt, int M, int K, int8_t *xq, float *beta,
                     int *rowsum, cudaStream_t st, int *clear = nullptr, int n_clear = 0,
                     const float *gain = nullptr, float eps = 0.0f)
{
    if (M == 0)
        return BITLINEAR_OK;
    const int row_bytes = K * (xdt == BITLINEAR_BF16 ? 2 : 4);
    const int rpb = std::min(qa::WARPS, kStagedQuantSmem / row_bytes);
    if (M >= kStagedQuantMinRows && rpb >= 4) {
        DeviceInfo *dev = nullptr;
        const int rc = current_device(&dev);
        if (rc != BITLINEAR_OK)
            return rc;
        return launch_qa_staged(x, xdt == BITLINEAR_BF16, M, K, rpb, xq, beta, rowsum, st, clear,
                                n_clear, gain, eps, dev->id);
    }
    const int nvec = K / 8;
    cudaError_t e;
    if (xdt == BITLINEAR_BF16) {
        if (nvec <= 32 * 4)
            e = launch_qa<true, 4, 1>(x, M, K, xq, beta, rowsum, st, clear, n_clear, gain, eps);
        else if (nvec <= 32 * 8)
            e = launch_qa<true, 8, 1>(x, M, K, xq, beta, rowsum, st, clear, n_clear, gain, eps);
        else if (nvec <= 32 * 16)
            e = launch_qa<true, 16, 1>(x, M, K, xq, beta, rowsum, st, clear, n_clear, gain, eps);
        else if (nvec <= 64 * 16)
            e = launch_qa<true, 16, 2>(x, M, K, xq, beta, rowsum, st, clear, n_clear, gain, eps);
        else if (nvec <= 128 * 16)
            e = launch_qa<true, 16, 4>(x, M, K, xq, beta, rowsum, st, clear, n_clear, gain, eps);
        else
            e = launch_qa<true, 16, 8>(x, M, K, xq, beta, rowsum, st, clear, n_clear, gain, eps);
    } else {
        if (nvec <= 32 * 4)
            e = launch_qa<false, 4, 1>(x, M, K, xq, beta, rowsum, st, clear, n_clear, gain, eps);
        else if (nvec <= 32 * 8)
            e = launch_qa<false, 8, 1>(x, M, K, xq, beta, rowsum, st, clear, n_clear, gain, eps);
        else if (nvec <= 64 * 8)
            e = launch_qa<false, 8, 2>(x, M, K, xq, beta, rowsum, st, clear, n_clear, gain, eps);
        else if (nvec <= 128 * 8)
            e = launch_qa<false, 8, 4>(x, M, K, xq, beta, rowsum, st, clear, n_clear, gain, eps);
        else
            e = launch_qa<false, 8, 8>(x, M, K, xq, beta, rowsum, st, clear, n_clear, gain, eps);
    }
    return launch_status(e);
}

// ------------------------------------------------------------------- GEMV

template <int MT, bool BF16, bool NORM, bool FFN, bool WIDE = false, bool B3 = false>
int launch_gemv_t(const gemv::Params &p, int grid, int smem, int dev, cudaStream_t st)
{
    cudaError_t e = allow_smem<gemv::gemv_kernel<MT, BF16, NORM, FFN, WIDE, B3>>(dev, smem);
    if (e != cudaSuccess)
        return launch_status(e);
    e = launch(gemv::gemv_kernel<MT, BF16, NORM, FFN, WIDE, B3>, dim3(grid), dim3(gemv::THREADS),
               smem, st, p);
    return launch_status(e);
}

// The kernels that read the base-3 layout.
template <int MT>
int launch_gemv_b3(const gemv::Params &p, bool bf16, int grid, int smem, int dev, cudaStream_t st)
{
    return bf16 ? launch_gemv_t<MT, true, false, false, false, true>(p, grid, smem, dev, st)
                : launch_gemv_t<MT, false, false, false, false, true>(p, grid, smem, dev, st);
}

template <int MT>
int launch_gemv_mt(const gemv::Params &p, bool bf16, bool norm, bool ffn, int grid, int smem,
                   int dev, cudaStream_t st)
{
    if (ffn) {
        if (norm)
            return bf16 ? launch_gemv_t<MT, true, true, true>(p, grid, smem, dev, st)
                        : launch_gemv_t<MT, false, true, true>(p, grid, smem, dev, st);
        return bf16 ? launch_gemv_t<MT, true, false, true>(p, grid, smem, dev, st)
                    : launch_gemv_t<MT, false, false, true>(p, grid, smem, dev, st);
    }
    if (norm)
        return bf16 ? launch_gemv_t<MT, true, true, false>(p, grid, smem, dev, st)
                    : launch_gemv_t<MT, false, true, false>(p, grid, smem, dev, st);
    return bf16 ? launch_gemv_t<MT, true, false, false>(p, grid, smem, dev, st)
                : launch_gemv_t<MT, false, false, false>(p, grid, smem, dev, st);
}

// The single-token bf16 kernel that stages a long row (8192 < K <= 32768) in
// shared memory for its prologue.
int launch_gemv_wide(const gemv::Params &p, int grid, int smem, int dev, cudaStream_t st)
{
    return launch_gemv_t<1, true, false, false, true>(p, grid, smem, dev, st);
}

// One problem of a GEMV launch, as the host sees it.
struct GemvJob {
    const void *x;
    int M, K, N;
    const void *packed;
    float gamma;
    void *y;
    int32_t *acc;
    int8_t *xq;
    float *beta;
    const float *norm_gain;     // non-null: RMS-normalise the tokens first
    float norm_eps;
    // the feed-forward form (one job per launch): the up projection, whose
    // rows pair with the gate rows above, and the output h
    const void *packed2 = nullptr;
    float gamma2 = 0.0f;
    const float *norm_gain2 = nullptr;
    void *y2 = nullptr;
    float *h = nullptr;
    bool b3 = false;            // `packed` is in the base-3 layout
};

// Launches the GEMV kernel over one or more independent problems. Every CTA
// owns whole 16-row blocks of one problem, about the same number of weight
// bytes in every CTA of the launch: the launch's bytes spread over two CTAs
// per SM, kept between 16 and 64 KiB per CTA, so large matrices run in
// several waves of small CTAs that the hardware balances over the SMs. Each
// CTA streams its blocks in chunks of up to QB blocks, a stage holding G
// k-groups of every block of the chunk (about 16 KiB). Either every problem
// of the launch is RMS-normalised or none is. With inject_timeout_us > 0 the
// producer leaves the first stage unloaded and every wait gives up after that
// many microseconds (the failure-detection test). A job with a non-null h is
// the feed-forward form (gate and up streamed together, h written); it is the
// launch's only job.
int launch_gemv(const GemvJob *jobs, int count, bitlinear_dtype xdt, const DeviceInfo &dev,
                cudaStream_t st, int inject_timeout_us = 0)
{
    const bool norm = jobs[0].norm_gain != nullptr;
    const bool ffn = jobs[0].h != nullptr;
    const bool b3 = jobs[0].b3;
    if (ffn && count != 1)
        return BITLINEAR_ERR_ARG;
    for (int i = 1; i < count; ++i)
        if (jobs[i].b3 != b3)
            return BITLINEAR_ERR_ARG;
    if (b3 && (norm || ffn))
        return BITLINEAR_ERR_ARG;
    // k-groups per row: of 128 weights, or of 160 in the base-3 layout, whose
    // rows (and the x~ rows) are padded to 160 per group
    auto groups_of = [b3](int K) { return b3 ? (K + 159) / 160 : K / 128; };
    auto xrow_of = [b3, &groups_of](int K) { return b3 ? groups_of(K) * 160 : K; };
    for (int i = 1; i < count; ++i)
        if ((jobs[i].norm_gain != nullptr) != norm)
            return BITLINEAR_ERR_ARG;
    int Mmax = 1;
    double total_bytes = 0.0;
    int xq_cap = 0;
    for (int i = 0; i < count; ++i) {
        Mmax = std::max(Mmax, jobs[i].M);
        total_bytes += static_cast<double>((jobs[i].N + 15) / 16) * groups_of(jobs[i].K) * 512.0;
        xq_cap = std::max(xq_cap, jobs[i].M * xrow_of(jobs[i].K));
    }
    const int MT = gemv_tile(Mmax);
    const int QB = gemv::chunk_blocks(MT, ffn);
    const int nmat = ffn ? 2 : 1;
    int max_K = 0;
    for (int i = 0; i < count; ++i)
        max_K = std::max(max_K, jobs[i].K);
    // one bf16 token of a long row: the wide kernel, whose x~ region first
    // holds the staged bf16 row (2 K bytes), two blocks per SM
    const bool wide = MT == 1 && !norm && !ffn && !b3 && xdt == BITLINEAR_BF16 && max_K > 8192 &&
                      max_K <= 32768;
    if (wide)
        xq_cap *= 2;
    int blocks[gemv::MAX_PROBLEMS], ctas[gemv::MAX_PROBLEMS], G[gemv::MAX_PROBLEMS];
    double bbytes[gemv::MAX_PROBLEMS];
    double max_block = 0.0;
    for (int i = 0; i < count; ++i) {
        blocks[i] = (jobs[i].N + 15) / 16;
        bbytes[i] = nmat * 512.0 * groups_of(jobs[i].K);
        max_block = std::max(max_block, bbytes[i]);
    }
    // CTAs: one wave of two per SM (a third fits beside them, for the next
    // kernel under programmatic dependent launch). One problem spreads its
    // blocks over min(blocks, 2 * SMs) CTAs, as evenly as whole blocks allow.
    // A group gives every CTA about the same bytes: each problem's CTAs hold at
    // most `target` bytes, the launch's bytes spread over two CTAs per SM (10%
    // slack, and at least one block), raised while the grid exceeds three CTAs
    // per SM.
    if (count == 1) {
        ctas[0] = std::min(blocks[0], 2 * dev.sms);
    } else {
        double target = std::max(max_block, 1.1 * total_bytes / (2.0 * dev.sms));
        for (int attempt = 0;; ++attempt) {
            int grid = 0;
            for (int i = 0; i < count; ++i) {
                const int q = std::max(1, static_cast<int>(target / bbytes[i]));
                ctas[i] = (blocks[i] + q - 1) / q;
                grid += ctas[i];
            }
            if (grid <= 3 * dev.sms || attempt > 64)
                break;
            target *= 1.25;
        }
    }
    int grid = 0;
    for (int i = 0; i < count; ++i)
        grid += ctas[i];
    // Stage geometry. When the whole rows of two or more blocks (or of a
    // CTA's only block) fit in a slot target (32 KiB), a chunk of cb blocks
    // streams as one contiguous copy per matrix (G = all K/128 groups);
    // otherwise a stage is a k-range of G groups (a multiple of 8, so that
    // each warp keeps its groups) of every block of the chunk, about 16 KiB,
    // one copy per block. Beside a large x~ the targets shrink.
    int cb[gemv::MAX_PROBLEMS];
    int target_rows = 32 * 1024, target_split = 16 * 1024;
    int slot_bytes = 0, slots = 0, red_blocks = 1, smem = 0;
    for (int attempt = 0;; ++attempt) {
        slot_bytes = 0;
        red_blocks = 1;
        int stages = 1;
        for (int i = 0; i < count; ++i) {
            const int KG = groups_of(jobs[i].K);
            const int q = (blocks[i] + ctas[i] - 1) / ctas[i];
            const int row_block = nmat * KG * gemv::PIECE;     // one block, all matrices
            if (2 * row_block <= target_rows || (q == 1 && row_block <= target_rows)) {
                cb[i] = std::max(1, std::min({QB, q, target_rows / row_block}));
                G[i] = KG;
            } else {
                cb[i] = std::min(q, QB);
                int g = std::max(8, (target_split / (nmat * cb[i] * gemv::PIECE)) & ~7);
                G[i] = g >= KG ? KG : g;
            }
            slot_bytes = std::max(slot_bytes, nmat * cb[i] * G[i] * gemv::PIECE);
            red_blocks = std::max(red_blocks, cb[i]);
            stages = std::max(stages, ((q + cb[i] - 1) / cb[i]) * ((KG + G[i] - 1) / G[i]));
        }
        // Ring depth: the whole share when it is small, else as deep as a
        // 72 KiB block allows (three blocks per SM fit beside each other, the
        // third for the next launch under programmatic dependent launch). A
        // stream of four or more stages per CTA (long rows, many blocks) and
        // the wide kernel get 110 KiB: two blocks per SM then keep more bytes
        // in flight, which a long stream needs more than the overlap with the
        // next launch (measured: 2B layer at B = 1 7.0 -> 6.4 us).
        const int fixed = gemv::smem_bytes(MT, xq_cap, 0, 0, red_blocks, norm, ffn, b3);
        const int ring_budget = (wide || stages >= 4) ? 110 * 1024 : 72 * 1024;
        slots = (ring_budget - fixed) / slot_bytes;
        slots = std::max(1, std::min({slots, stages, gemv::MAX_SLOTS}));
        if (stages > 1)
            slots = std::max(slots, 2);
        smem = gemv::smem_bytes(MT, xq_cap, slots, slot_bytes, red_blocks, norm, ffn, b3);
        if (smem <= dev.max_smem_optin)
            break;
        // too large beside a large x~: smaller stages
        if (attempt >= 8 || (target_rows <= 4096 && target_split <= 4096))
            return BITLINEAR_ERR_SHAPE;
        target_rows = std::max(4096, target_rows / 2);
        target_split = std::max(4096, target_split / 2);
    }
    gemv::Params p = {};
    int begin = 0;
    for (int i = 0; i < count; ++i) {
        const GemvJob &j = jobs[i];
        p.prob[i] = gemv::Problem{j.x,
                                  static_cast<const uint8_t *>(j.packed),
                                  static_cast<uint16_t *>(j.y),
                                  j.acc,
                                  j.xq,
                                  j.beta,
                                  j.M,
                                  j.K,
                                  j.N,
                                  j.gamma,
                                  j.norm_gain,
                                  j.norm_eps,
                                  blocks[i] / ctas[i],
                                  blocks[i] % ctas[i],
                                  begin,
                                  cb[i],
                                  G[i],
                                  static_cast<const uint8_t *>(j.packed2),
                                  j.gamma2,
                                  j.norm_gain2,
                                  static_cast<uint16_t *>(j.y2),
                                  j.h};
        begin += ctas[i];
    }
    p.count = count;
    p.slots = slots;
    p.slot_bytes = slot_bytes;
    p.xq_cap = xq_cap;
    p.red_blocks = red_blocks;
    p.wait_limit_ns = inject_timeout_us > 0 ? static_cast<uint64_t>(inject_timeout_us) * 1000ull
                                            : kWaitLimitNs;
    p.inject_timeout = inject_timeout_us > 0 ? 1 : 0;
    const bool bf16 = xdt == BITLINEAR_BF16;
    if (wide)
        return launch_gemv_wide(p, grid, smem, dev.id, st);
    if (b3) {
        switch (MT) {
        case 1: return launch_gemv_b3<1>(p, bf16, grid, smem, dev.id, st);
        case 2: return launch_gemv_b3<2>(p, bf16, grid, smem, dev.id, st);
        case 4: return launch_gemv_b3<4>(p, bf16, grid, smem, dev.id, st);
        case 8: return launch_gemv_b3<8>(p, bf16, grid, smem, dev.id, st);
        default: return launch_gemv_b3<16>(p, bf16, grid, smem, dev.id, st);
        }
    }
    switch (MT) {
    case 1: return launch_gemv_mt<1>(p, bf16, norm, ffn, grid, smem, dev.id, st);
    case 2: return launch_gemv_mt<2>(p, bf16, norm, ffn, grid, smem, dev.id, st);
    case 4: return launch_gemv_mt<4>(p, bf16, norm, ffn, grid, smem, dev.id, st);
    case 8: return launch_gemv_mt<8>(p, bf16, norm, ffn, grid, smem, dev.id, st);
    default: return launch_gemv_mt<16>(p, bf16, norm, ffn, grid, smem, dev.id, st);
    }
}

// ------------------------------------------------------------ tensor cores

// Token tile of the weight-stationary GEMM: the candidate that pads M the
// least (ties go to the larger tile).
int choose_bt(int64_t M)
{
    if (M <= 32)
        return 32;
    if (M <= 64)
        return 64;
    if (M <= 128)
        return 128;
    const int64_t pad128 = (M + 127) / 128 * 128;
    const int64_t pad192 = (M + 191) / 192 * 192;
    return pad192 <= pad128 ? 192 : 128;
}

// x~, beta and the row sums of x~ of one problem.
size_t tc_base_bytes(int64_t M, int64_t K)
{
    return round_up(static_cast<size_t>(M) * static_cast<size_t>(K), 256) +
           2 * round_up(static_cast<size_t>(M) * 4, 256);
}

// Flags and partial-sum slots for tiles split between CTAs.
size_t tc_split_bytes(int64_t max_M)
{
    return round_up(static_cast<size_t>(wsg::MAX_GRID) * 4 * 4, 256) +
           static_cast<size_t>(wsg::MAX_GRID) * wsg::BW * static_cast<size_t>(choose_bt(max_M)) * 4;
}

size_t tc_workspace_bytes(int64_t M, int64_t K) { return tc_base_bytes(M, K) + tc_split_bytes(M); }

// One problem of a tensor-core launch, as the host sees it.
struct TcJob {
    const void *x;
    int M, K, N;
    const void *packed;
    float gamma;
    void *y;
    int32_t *acc;
    const float *norm_gain;     // non-null: RMS-normalise the tokens first (single problem)
    float norm_eps;
};

size_t tc_group_bytes(const TcJob *jobs, int n, bool split)
{
    size_t b = 0;
    int max_M = 0;
    for (int i = 0; i < n; ++i) {
        b += tc_base_bytes(jobs[i].M, jobs[i].K);
        max_M = std::max(max_M, jobs[i].M);
    }
    return b + (split ? tc_split_bytes(max_M) : 0);
}

template <int BT, int BK = 256>
int launch_gemm_ws(const wsg::Maps &maps, const wsg::Params &p, int grid, const DeviceInfo &dev,
                   cudaStream_t st)
{
    constexpr int smem = wsg::Cfg<BT, BK>::SMEM_BYTES;
    cudaError_t e = allow_smem<wsg::gemm_ws_kernel<BT, BK>>(dev.id, smem);
    if (e != cudaSuccess)
        return launch_status(e);
    e = launch(wsg::gemm_ws_kernel<BT, BK>, dim3(grid), dim3(wsg::Cfg<BT, BK>::THREADS),
               static_cast<size_t>(smem), st, maps, p);
    return launch_status(e);
}

// Quantisation of several problems' rows in one launch (WPR warps per row),
// RMS-normalising each problem's rows with its own gains when they are given
// (all problems or none).
template <bool BF16, int CACHE, int WPR>
cudaError_t launch_qa_group(const TcJob *jobs, int n, int8_t *const *xq, float *const *beta,
                            int *const *rowsum, cudaStream_t st, int *clear, int n_clear)
{
    constexpr int rpb = qa::rows_per_block<WPR>();
    qa::GroupParams g{};
    int blocks = 0;
    for (int i = 0; i < n; ++i) {
        g.prob[i] = qa::GroupRows{jobs[i].x,        xq[i],    beta[i], rowsum[i],
                                  jobs[i].M,        jobs[i].K, blocks, jobs[i].norm_gain,
                                  jobs[i].norm_eps};
        blocks += (jobs[i].M + rpb - 1) / rpb;
    }
    g.count = n;
    g.clear = clear;
    g.n_clear = n_clear;
    if (jobs[0].norm_gain != nullptr)
        return launch(qa::quant_act_grouped_kernel<BF16, CACHE, WPR, true>, dim3(blocks),
                      dim3(qa::THREADS), 0, st, g);
    return launch(qa::quant_act_grouped_kernel<BF16, CACHE, WPR, false>, dim3(blocks),
                  dim3(qa::THREADS), 0, st, g);
}

// Warps per row chosen by the group's longest row, as for one problem.
int launch_quant_group(const TcJob *jobs, int n, bitlinear_dtype xdt, int8_t *const *xq,
                       float *const *beta, int *const *rowsum, cudaStream_t st, int *clear,
                       int n_clear)
{
    int max_K = 0;
    for (int i = 0; i < n; ++i)
        max_K = std::max(max_K, jobs[i].K);
    const int nvec = max_K / 8;
    cudaError_t e;
    if (xdt == BITLINEAR_BF16) {
        if (nvec <= 32 * 16)
            e = launch_qa_group<true, 16, 1>(jobs, n, xq, beta, rowsum, st, clear, n_clear);
        else if (nvec <= 64 * 16)
            e = launch_qa_group<true, 16, 2>(jobs, n, xq, beta, rowsum, st, clear, n_clear);
        else
            e = launch_qa_group<true, 16, 8>(jobs, n, xq, beta, rowsum, st, clear, n_clear);
    } else {
        if (nvec <= 32 * 8)
            e = launch_qa_group<false, 8, 1>(jobs, n, xq, beta, rowsum, st, clear, n_clear);
        else if (nvec <= 64 * 8)
            e = launch_qa_group<false, 8, 2>(jobs, n, xq, beta, rowsum, st, clear, n_clear);
        else
            e = launch_qa_group<false, 8, 8>(jobs, n, xq, beta, rowsum, st, clear, n_clear);
    }
    return launch_status(e);
}

// Quantise x, then run the weight-stationary GEMM with its fused rescale, for
// one or several independent problems (at most wsg::MAX_PROBLEMS) in one pair
// of launches. The workspace holds each problem's x~, beta and row sums, then
// (with `split`) the flag and partial-sum regions. With `split` the k-blocks
// of all tiles are shared evenly between the CTAs (stream-K) when that pays;
// otherwise every CTA takes whole tiles.
int run_tc_group(const TcJob *jobs, int n, bitlinear_dtype xdt, void *ws, size_t ws_bytes,
                 int8_t *xq_dbg, float *beta_dbg, const DeviceInfo &dev, cudaStream_t st,
                 int inject_timeout_us, bool split)
{
    const size_t need = tc_group_bytes(jobs, n, split);
    if (ws == nullptr || ws_bytes < need)
        return BITLINEAR_ERR_WORKSPACE;
    for (int i = 1; i < n; ++i)                   // normalise every problem or none
        if ((jobs[i].norm_gain != nullptr) != (jobs[0].norm_gain != nullptr))
            return BITLINEAR_ERR_ARG;
    if (!aligned(ws, 256))
        return BITLINEAR_ERR_ALIGN;
    int max_M = 0;
    for (int i = 0; i < n; ++i)
        max_M = std::max(max_M, jobs[i].M);
    const int BT = choose_bt(max_M);
    const int slots = std::min(dev.sms, wsg::MAX_GRID);
    // Stage depth: 512 k for the small token tiles when every CTA has at
    // least kDeepStageMinBlocks k-blocks of 256 to stream (deep_stages_fit).
    int64_t iters256 = 0;
    for (int i = 0; i < n; ++i)
        iters256 += static_cast<int64_t>((jobs[i].M + BT - 1) / BT) *
                    ((jobs[i].N + wsg::BW - 1) / wsg::BW) * ((jobs[i].K + 255) / 256);
    const int BK =
        (wsg::deep_stages_fit(BT) && iters256 >= kDeepStageMinBlocks * slots) ? 512 : 256;

    wsg::Params p{};
    int64_t tiles = 0, iters = 0;
    for (int i = 0; i < n; ++i) {
        wsg::Problem &P = p.prob[i];
        P.M = jobs[i].M;
        P.N = jobs[i].N;
        P.MT = (jobs[i].M + BT - 1) / BT;
        P.KB = (jobs[i].K + BK - 1) / BK;
        P.iter_begin = static_cast<int>(iters);
        P.tile_begin = static_cast<int>(tiles);
        P.gamma = jobs[i].gamma;
        P.y = static_cast<uint16_t *>(jobs[i].y);
        P.acc_out = jobs[i].acc;
        const int64_t T = static_cast<int64_t>(P.MT) * ((jobs[i].N + wsg::BW - 1) / wsg::BW);
        tiles += T;
        iters += T * P.KB;
    }
    if (iters >= (int64_t(1) << 31))
        return BITLINEAR_ERR_SHAPE;
    // Splitting a tile's k-range between CTAs costs a hand-off of a few
    // microseconds (partial store, flag, partial load). With at least as many
    // tiles as CTAs it evens out the last wave; with fewer tiles it pays only
    // when the k-blocks a CTA saves outweigh that hand-off.
    if (split && tiles < slots) {
        const double kb_per_tile = static_cast<double>(iters) / static_cast<double>(tiles);
        const double saved_blocks = kb_per_tile * (1.0 - static_cast<double>(tiles) / slots);
        // in 256-k blocks, whatever the launch's stage depth
        split = saved_blocks * (BK / 256) > kSplitMinSavedBlocks;
    }
    const int64_t units = split ? iters : tiles;
    int64_t grid64 = std::min<int64_t>(units, slots);
    if (split && tiles < slots)
        grid64 = std::max<int64_t>(
            tiles, std::min<int64_t>(grid64, iters * (BK / 256) / kSplitMinCtaBlocks));
    const int grid = static_cast<int>(grid64);

    // Workspace: per problem x~ | beta | row sums, then flags | partial sums.
    char *w = static_cast<char *>(ws);
    int8_t *xq[wsg::MAX_PROBLEMS];
    float *beta[wsg::MAX_PROBLEMS];
    int *rowsum[wsg::MAX_PROBLEMS];
    for (int i = 0; i < n; ++i) {
        const size_t a = round_up(static_cast<size_t>(jobs[i].M) * jobs[i].K, 256);
        const size_t c = round_up(static_cast<size_t>(jobs[i].M) * 4, 256);
        xq[i] = reinterpret_cast<int8_t *>(w);
        beta[i] = reinterpret_cast<float *>(w + a);
        rowsum[i] = reinterpret_cast<int *>(w + a + c);
        p.prob[i].beta = beta[i];
        p.prob[i].rowsum = rowsum[i];
        w += a + 2 * c;
    }
    int *flags = nullptr;
    if (split) {
        flags = reinterpret_cast<int *>(w);
        p.partial = reinterpret_cast<int32_t *>(
            w + round_up(static_cast<size_t>(wsg::MAX_GRID) * 4 * 4, 256));
        p.flags = flags;
    }
    int rc = (n == 1) ? launch_quant_act(jobs[0].x, xdt, jobs[0].M, jobs[0].K, xq[0], beta[0],
                                         rowsum[0], st, flags, split ? 4 * grid : 0,
                                         jobs[0].norm_gain, jobs[0].norm_eps)
                      : launch_quant_group(jobs, n, xdt, xq, beta, rowsum, st, flags,
                                           split ? 4 * grid : 0);
    if (rc != BITLINEAR_OK)
        return rc;
    wsg::Maps maps{};
    for (int i = 0; i < n; ++i)
        if (!make_map_xq(&maps.x[i], xq[i], jobs[i].M, jobs[i].K, static_cast<uint32_t>(BT),
                         static_cast<uint32_t>(BK / wsg::SUB_K)) ||
            !make_map_packed(&maps.w[i], jobs[i].packed, jobs[i].N, jobs[i].K, wsg::BW,
                             static_cast<uint32_t>(BK / wsg::SUB_K)))
            return BITLINEAR_ERR_CUDA;
    p.count = n;
    p.total_iters = static_cast<int>(iters);
    p.total_tiles = static_cast<int>(tiles);
    p.split = split ? 1 : 0;
    p.base = static_cast<int>(units / grid);
    p.extra = static_cast<int>(units % grid);
    p.wait_limit_ns =
        inject_timeout_us > 0 ? static_cast<uint64_t>(inject_timeout_us) * 1000ull : kWaitLimitNs;
    p.inject_timeout = inject_timeout_us > 0 ? 1 : 0;
    switch (BT) {
    case 32:
        rc = BK == 512 ? launch_gemm_ws<32, 512>(maps, p, grid, dev, st)
                       : launch_gemm_ws<32>(maps, p, grid, dev, st);
        break;
    case 64:
        rc = BK == 512 ? launch_gemm_ws<64, 512>(maps, p, grid, dev, st)
                       : launch_gemm_ws<64>(maps, p, grid, dev, st);
        break;
    case 128: rc = launch_gemm_ws<128>(maps, p, grid, dev, st); break;
    default: rc = launch_gemm_ws<192>(maps, p, grid, dev, st); break;
    }
    if (rc != BITLINEAR_OK)
        return rc;
    if (n == 1 && xq_dbg != nullptr &&
        cudaMemcpyAsync(xq_dbg, xq[0], static_cast<size_t>(jobs[0].M) * jobs[0].K,
                        cudaMemcpyDeviceToDevice, st) != cudaSuccess)
        return BITLINEAR_ERR_CUDA;
    if (n == 1 && beta_dbg != nullptr &&
        cudaMemcpyAsync(beta_dbg, beta[0], static_cast<size_t>(jobs[0].M) * 4,
                        cudaMemcpyDeviceToDevice, st) != cudaSuccess)
        return BITLINEAR_ERR_CUDA;
    return BITLINEAR_OK;
}

int run_tc_path(const void *x, bitlinear_dtype xdt, int M, int K, const void *packed,
                float gamma, int N, void *y, void *ws, size_t ws_bytes, int32_t *acc,
                int8_t *xq_dbg, float *beta_dbg, const DeviceInfo &dev, cudaStream_t st,
                int inject_timeout_us, bool split, const float *norm_gain = nullptr,
                float norm_eps = 0.0f)
{
    const TcJob job{x, M, K, N, packed, gamma, y, acc, norm_gain, norm_eps};
    return run_tc_group(&job, 1, xdt, ws, ws_bytes, xq_dbg, beta_dbg, dev, st, inject_timeout_us,
                        split);
}

// --------------------------------------------------------------- checks

int check_forward_args(const void *x, int xdt, int64_t M, int64_t K, const void *packed,
                       int64_t N, const void *y, const int32_t *acc, const int8_t *xq,
                       const float *beta)
{
    if (M < 0 || N < 1 || K < 1)
        return BITLINEAR_ERR_ARG;
    if (M > 0 && (x == nullptr || packed == nullptr || y == nullptr))
        return BITLINEAR_ERR_ARG;
    if (xdt != BITLINEAR_BF16 && xdt != BITLINEAR_FP32)
        return BITLINEAR_ERR_DTYPE;
    if (K % 128 != 0 || K > kMaxK || N > INT_MAX / 2 || M > INT_MAX / 2 ||
        M * K > (int64_t(1) << 40))
        return BITLINEAR_ERR_SHAPE;
    if (!aligned(x, 16) || !aligned(packed, 16) || !aligned(y, 16) || !aligned(xq, 16) ||
        !aligned(acc, 4) || !aligned(beta, 4))
        return BITLINEAR_ERR_ALIGN;
    return BITLINEAR_OK;
}


int choose_path(int64_t M, int64_t K, int path)
{
    if (path == BITLINEAR_PATH_GEMV || path == BITLINEAR_PATH_TC)
        return path;
    return (M <= kAutoGemvMaxM && gemv_fits(M, K)) ? BITLINEAR_PATH_GEMV : BITLINEAR_PATH_TC;
}

int forward_impl(const void *x, bitlinear_dtype xdt, int64_t M, int64_t K, const void *packed,
                 float gamma, int64_t N, void *y, void *ws, size_t ws_bytes, void *stream,
                 int32_t *acc, int8_t *xq, float *beta, int path, int inject_timeout_us,
                 const float *norm_gain = nullptr, float norm_eps = 0.0f)
{
    int rc = check_forward_args(x, xdt, M, K, packed, N, y, acc, xq, beta);
    if (rc != BITLINEAR_OK)
        return rc;
    if (path < BITLINEAR_PATH_AUTO || path > BITLINEAR_PATH_TC)
        return BITLINEAR_ERR_ARG;
    if (M == 0)
        return BITLINEAR_OK;
    const int chosen = choose_path(M, K, path);
    if (chosen == BITLINEAR_PATH_GEMV && !gemv_fits(M, K))
        return BITLINEAR_ERR_SHAPE;
    DeviceInfo *dev = nullptr;
    rc = current_device(&dev);
    if (rc != BITLINEAR_OK)
        return rc;
    cudaStream_t st = static_cast<cudaStream_t>(stream);
    if (chosen == BITLINEAR_PATH_GEMV) {
        const GemvJob job{x,      static_cast<int>(M), static_cast<int>(K), static_cast<int>(N),
                          packed, gamma, y, acc, xq, beta, norm_gain, norm_eps};
        return launch_gemv(&job, 1, xdt, *dev, st, inject_timeout_us);
    }
    return run_tc_path(x, xdt, static_cast<int>(M), static_cast<int>(K), packed, gamma,
                       static_cast<int>(N), y, ws, ws_bytes, acc, xq, beta, *dev, st,
                       inject_timeout_us, true, norm_gain, norm_eps);
}

}  // namespace

// ================================================================== C ABI

extern "C" const char *bitlinear_status_string(int status)
{
    switch (status) {
    case BITLINEAR_OK: return "ok";
    case BITLINEAR_ERR_ARG: return "invalid argument";
    case BITLINEAR_ERR_SHAPE: return "unsupported shape";
    case BITLINEAR_ERR_ALIGN: return "misaligned pointer";
    case BITLINEAR_ERR_DTYPE: return "unsupported dtype";
    case BITLINEAR_ERR_CUDA: return "CUDA error";
    case BITLINEAR_ERR_TIMEOUT: return "device wait timed out";
    case BITLINEAR_ERR_WORKSPACE: return "workspace missing or too small";
    case BITLINEAR_ERR_SCRATCH_LIMIT: return "problem exceeds the static scratch limit";
    case BITLINEAR_ERR_HOST: return "host allocation failed";
    case BITLINEAR_ERR_IO: return "file could not be read or written";
    case BITLINEAR_ERR_FORMAT: return "not a valid packed-weight file";
    default: return "unknown status";
    }
}

extern "C" int bitlinear_quant_act(const void *x_dev, bitlinear_dtype xdt, int64_t M, int64_t K,
                                   int8_t *xq_dev, float *beta_dev, void *cuda_stream)
{
    if (M < 0 || K < 1)
        return BITLINEAR_ERR_ARG;
    if (M > 0 && (x_dev == nullptr || xq_dev == nullptr || beta_dev == nullptr))
        return BITLINEAR_ERR_ARG;
    if (xdt != BITLINEAR_BF16 && xdt != BITLINEAR_FP32)
        return BITLINEAR_ERR_DTYPE;
    if (K % 128 != 0 || K > (int64_t(1) << 30) || M > INT_MAX)
        return BITLINEAR_ERR_SHAPE;
    if (!aligned(x_dev, 16) || !aligned(xq_dev, 16) || !aligned(beta_dev, 4))
        return BITLINEAR_ERR_ALIGN;
    return launch_quant_act(x_dev, xdt, static_cast<int>(M), static_cast<int>(K), xq_dev,
                            beta_dev, nullptr, static_cast<cudaStream_t>(cuda_stream));
}

extern "C" size_t bitlinear_workspace_bytes_path(int64_t M, int64_t N, int64_t K, int path)
{
    if (M < 0 || N < 1 || K < 1 || K % 128 != 0 || K > kMaxK)
        return SIZE_MAX;
    if (path < BITLINEAR_PATH_AUTO || path > BITLINEAR_PATH_TC)
        return SIZE_MAX;
    if (M == 0)
        return 0;
    if (path == BITLINEAR_PATH_GEMV && !gemv_fits(M, K))
        return SIZE_MAX;                          // the GEMV cannot take this shape
    return choose_path(M, K, path) == BITLINEAR_PATH_GEMV ? 0 : tc_workspace_bytes(M, K);
}

extern "C" size_t bitlinear_workspace_bytes(int64_t M, int64_t N, int64_t K)
{
    return bitlinear_workspace_bytes_path(M, N, K, BITLINEAR_PATH_AUTO);
}

extern "C" int bitlinear_forward(const void *x_dev, bitlinear_dtype xdt, int64_t M, int64_t K,
                                 const void *packed_dev, float gamma, int64_t N, void *y_dev,
                                 void *workspace_dev, size_t workspace_bytes, void *cuda_stream,
                                 int32_t *acc_dev_or_null, int8_t *xq_dev_or_null,
                                 float *beta_dev_or_null)
{
    return forward_impl(x_dev, xdt, M, K, packed_dev, gamma, N, y_dev, workspace_dev,
                        workspace_bytes, cuda_stream, acc_dev_or_null, xq_dev_or_null,
                        beta_dev_or_null, BITLINEAR_PATH_AUTO, 0);
}

extern "C" int bitlinear_forward_ex(const void *x_dev, bitlinear_dtype xdt, int64_t M, int64_t K,
                                    const void *packed_dev, float gamma, int64_t N, void *y_dev,
                                    void *workspace_dev, size_t workspace_bytes,
                                    void *cuda_stream, int32_t *acc_dev_or_null,
                                    int8_t *xq_dev_or_null, float *beta_dev_or_null, int path)
{
    return forward_impl(x_dev, xdt, M, K, packed_dev, gamma, N, y_dev, workspace_dev,
                        workspace_bytes, cuda_stream, acc_dev_or_null, xq_dev_or_null,
                        beta_dev_or_null, path, 0);
}

extern "C" int bitlinear_forward_rmsnorm(const void *x_dev, bitlinear_dtype xdt, int64_t M,
                                         int64_t K, const float *norm_gain_dev, float norm_eps,
                                         const void *packed_dev, float gamma, int64_t N,
                                         void *y_dev, void *workspace_dev, size_t workspace_bytes,
                                         void *cuda_stream, int32_t *acc_dev_or_null,
                                         int8_t *xq_dev_or_null, float *beta_dev_or_null,
                                         int path)
{
    if (M > 0 && norm_gain_dev == nullptr)
        return BITLINEAR_ERR_ARG;
    if (!(norm_eps > 0.0f) || !(norm_eps <= FLT_MAX))
        return BITLINEAR_ERR_ARG;
    if (!aligned(norm_gain_dev, 16))
        return BITLINEAR_ERR_ALIGN;
    // M = 0 stays a no-op, which needs no gains
    const float *gain = M > 0 ? norm_gain_dev : nullptr;
    return forward_impl(x_dev, xdt, M, K, packed_dev, gamma, N, y_dev, workspace_dev,
                        workspace_bytes, cuda_stream, acc_dev_or_null, xq_dev_or_null,
                        beta_dev_or_null, path, 0, gain, norm_eps);
}

namespace {

// Argument checks of the feed-forward calls that do not depend on pointers:
// returns BITLINEAR_OK when (M, K, F) and the gains' presence are acceptable.
int check_ffn_shape(int64_t M, int64_t K, int64_t F)
{
    if (M < 0 || K < 1 || F < 1)
        return BITLINEAR_ERR_ARG;
    if (K % 128 != 0 || F % 128 != 0 || K > kMaxK || F > kMaxK || M > INT_MAX / 2 ||
        M * K > (int64_t(1) << 40) || M * F > (int64_t(1) << 40))
        return BITLINEAR_ERR_SHAPE;
    return BITLINEAR_OK;
}

// The fused GEMV launch takes the gate and up projections for decode batches
// (the automatic GEMV threshold) whose quantised tokens fit beside it (two
// copies when both projections normalise with their own gains); other
// batches take the tensor-core route.
bool ffn_fused(int64_t M, int64_t K, bool gate_up_norm)
{
    return M <= kAutoGemvMaxM && (gate_up_norm ? 2 : 1) * M * K <= gemv_max_xq(M);
}

// Workspace of the tensor-core route: the grouped gate/up launch's scratch
// (*group_bytes) and its two bf16 outputs (*out_bytes each), then, reusing
// all of it once they are consumed (stream order), the down projection's.
size_t ffn_tc_bytes(int64_t M, int64_t K, int64_t F, size_t *group_bytes = nullptr,
                    size_t *out_bytes = nullptr)
{
    TcJob jobs[2] = {};
    for (TcJob &j : jobs) {
        j.M = static_cast<int>(M);
        j.K = static_cast<int>(K);
        j.N = static_cast<int>(F);
    }
    const size_t g = tc_group_bytes(jobs, 2, true);
    const size_t o = round_up(static_cast<size_t>(M) * static_cast<size_t>(F) * 2, 256);
    if (group_bytes != nullptr)
        *group_bytes = g;
    if (out_bytes != nullptr)
        *out_bytes = o;
    return std::max(g + 2 * o, bitlinear_workspace_bytes_path(M, K, F, BITLINEAR_PATH_AUTO));
}

}  // namespace

extern "C" size_t bitlinear_workspace_bytes_ffn(int64_t M, int64_t K, int64_t F)
{
    if (check_ffn_shape(M, K, F) != BITLINEAR_OK)
        return SIZE_MAX;
    // without knowing the gains: the route that normalised gate/up inputs
    // would take sets the size
    if (ffn_fused(M, K, true))
        return bitlinear_workspace_bytes_path(M, K, F, BITLINEAR_PATH_AUTO);
    return ffn_tc_bytes(M, K, F);
}

extern "C" int bitlinear_ffn_forward(const void *x_dev, bitlinear_dtype xdt, int64_t M, int64_t K,
                                     int64_t F, const void *gate_packed_dev, float gate_gamma,
                                     const void *up_packed_dev, float up_gamma,
                                     const void *down_packed_dev, float down_gamma,
                                     const float *gate_gain_dev, const float *up_gain_dev,
                                     const float *down_gain_dev, float norm_eps, float *h_dev,
                                     void *y_dev, void *workspace_dev, size_t workspace_bytes,
                                     void *cuda_stream, void *gate_y_dev_or_null,
                                     void *up_y_dev_or_null)
{
    if ((gate_gain_dev == nullptr) != (up_gain_dev == nullptr))
        return BITLINEAR_ERR_ARG;
    const bool gu_norm = gate_gain_dev != nullptr;
    int rc = check_ffn_shape(M, K, F);
    if (rc != BITLINEAR_OK)
        return rc;
    if (xdt != BITLINEAR_BF16 && xdt != BITLINEAR_FP32)
        return BITLINEAR_ERR_DTYPE;
    if ((gu_norm || down_gain_dev != nullptr) && (!(norm_eps > 0.0f) || !(norm_eps <= FLT_MAX)))
        return BITLINEAR_ERR_ARG;
    if (M == 0)
        return BITLINEAR_OK;
    if (x_dev == nullptr || gate_packed_dev == nullptr || up_packed_dev == nullptr ||
        down_packed_dev == nullptr || h_dev == nullptr || y_dev == nullptr)
        return BITLINEAR_ERR_ARG;
    if (!aligned(x_dev, 16) || !aligned(gate_packed_dev, 16) || !aligned(up_packed_dev, 16) ||
        !aligned(down_packed_dev, 16) || !aligned(h_dev, 16) || !aligned(y_dev, 16) ||
        !aligned(gate_gain_dev, 16) || !aligned(up_gain_dev, 16) || !aligned(down_gain_dev, 16) ||
        !aligned(gate_y_dev_or_null, 16) || !aligned(up_y_dev_or_null, 16))
        return BITLINEAR_ERR_ALIGN;
    const bool fused = ffn_fused(M, K, gu_norm);
    // the down projection's own checks (workspace included) before any launch
    const int down_path = choose_path(M, F, BITLINEAR_PATH_AUTO);
    if (down_path == BITLINEAR_PATH_TC &&
        (workspace_dev == nullptr || workspace_bytes < tc_workspace_bytes(M, F)))
        return BITLINEAR_ERR_WORKSPACE;
    if (!fused && (workspace_dev == nullptr || workspace_bytes < ffn_tc_bytes(M, K, F)))
        return BITLINEAR_ERR_WORKSPACE;
    if (!fused && !aligned(workspace_dev, 256))
        return BITLINEAR_ERR_ALIGN;
    DeviceInfo *dev = nullptr;
    rc = current_device(&dev);
    if (rc != BITLINEAR_OK)
        return rc;
    cudaStream_t st = static_cast<cudaStream_t>(cuda_stream);
    if (!fused) {
        // Tensor-core route: gate and up as one grouped launch pair (each
        // with its own gains), h from their bf16 outputs, then the down
        // projection, which reuses the whole workspace.
        size_t group_bytes = 0, out_bytes = 0;
        ffn_tc_bytes(M, K, F, &group_bytes, &out_bytes);
        char *w = static_cast<char *>(workspace_dev);
        void *gy = gate_y_dev_or_null != nullptr ? gate_y_dev_or_null : w + group_bytes;
        void *uy = up_y_dev_or_null != nullptr ? up_y_dev_or_null : w + group_bytes + out_bytes;
        TcJob jobs[2] = {};
        const void *packs[2] = {gate_packed_dev, up_packed_dev};
        const float gammas[2] = {gate_gamma, up_gamma};
        const float *gains[2] = {gate_gain_dev, up_gain_dev};
        void *outs[2] = {gy, uy};
        for (int i = 0; i < 2; ++i)
            jobs[i] = TcJob{x_dev, static_cast<int>(M), static_cast<int>(K), static_cast<int>(F),
                            packs[i], gammas[i], outs[i], nullptr, gains[i], norm_eps};
        rc = run_tc_group(jobs, 2, xdt, workspace_dev, group_bytes, nullptr, nullptr, *dev, st, 0,
                          true);
        if (rc != BITLINEAR_OK)
            return rc;
        const int64_t n8 = M * F / 8;
        const int grid = static_cast<int>(
            std::max<int64_t>(1, std::min<int64_t>((n8 + ffn::THREADS - 1) / ffn::THREADS,
                                                   2 * dev->sms)));
        rc = launch_status(launch(ffn::relu2_glu_kernel, dim3(grid), dim3(ffn::THREADS), 0, st,
                                  static_cast<const uint16_t *>(gy),
                                  static_cast<const uint16_t *>(uy), h_dev, n8));
        if (rc != BITLINEAR_OK)
            return rc;
        return forward_impl(h_dev, BITLINEAR_FP32, M, F, down_packed_dev, down_gamma, K, y_dev,
                            workspace_dev, workspace_bytes, cuda_stream, nullptr, nullptr,
                            nullptr, BITLINEAR_PATH_AUTO, 0, down_gain_dev, norm_eps);
    }
    GemvJob job{x_dev,
                static_cast<int>(M),
                static_cast<int>(K),
                static_cast<int>(F),
                gate_packed_dev,
                gate_gamma,
                gate_y_dev_or_null,
                nullptr,
                nullptr,
                nullptr,
                gate_gain_dev,
                norm_eps};
    job.packed2 = up_packed_dev;
    job.gamma2 = up_gamma;
    job.norm_gain2 = up_gain_dev;
    job.y2 = up_y_dev_or_null;
    job.h = h_dev;
    rc = launch_gemv(&job, 1, xdt, *dev, st);
    if (rc != BITLINEAR_OK)
        return rc;
    return forward_impl(h_dev, BITLINEAR_FP32, M, F, down_packed_dev, down_gamma, K, y_dev,
                        workspace_dev, workspace_bytes, cuda_stream, nullptr, nullptr, nullptr,
                        BITLINEAR_PATH_AUTO, 0, down_gain_dev, norm_eps);
}

extern "C" int bitlinear_forward_b3(const void *x_dev, bitlinear_dtype xdt, int64_t M, int64_t K,
                                    const void *packed_b3_dev, float gamma, int64_t N,
                                    void *y_dev, void *cuda_stream, int32_t *acc_dev_or_null,
                                    int8_t *xq_dev_or_null, float *beta_dev_or_null)
{
    int rc = check_forward_args(x_dev, xdt, M, K, packed_b3_dev, N, y_dev, acc_dev_or_null,
                                xq_dev_or_null, beta_dev_or_null);
    if (rc != BITLINEAR_OK)
        return rc;
    if (M == 0)
        return BITLINEAR_OK;
    // the GEMV holds the tokens' x~ rows, padded to 160-weight groups
    const int64_t Kp = (K + 159) / 160 * 160;
    if (M > kGemvMaxM || M * Kp > gemv_max_xq(M))
        return BITLINEAR_ERR_SHAPE;
    DeviceInfo *dev = nullptr;
    rc = current_device(&dev);
    if (rc != BITLINEAR_OK)
        return rc;
    GemvJob job{x_dev,
                static_cast<int>(M),
                static_cast<int>(K),
                static_cast<int>(N),
                packed_b3_dev,
                gamma,
                y_dev,
                acc_dev_or_null,
                xq_dev_or_null,
                beta_dev_or_null,
                nullptr,
                0.0f};
    job.b3 = true;
    return launch_gemv(&job, 1, xdt, *dev, static_cast<cudaStream_t>(cuda_stream));
}

namespace {

// Checks a problem list for the one-launch grouped GEMV and collects its
// non-empty problems into jobs[0 .. *n). With b3 the weights are in the
// base-3 layout, whose x~ rows the GEMV pads to 160-weight groups.
int collect_gemv_group(const bitlinear_problem *problems, int count, bitlinear_dtype xdt,
                       GemvJob *jobs, int *n, bool b3 = false)
{
    if (problems == nullptr || count < 1 || count > gemv::MAX_PROBLEMS)
        return BITLINEAR_ERR_ARG;
    *n = 0;
    int64_t max_M = 0, max_xq = 0;
    for (int i = 0; i < count; ++i) {
        const bitlinear_problem &pr = problems[i];
        int rc = check_forward_args(pr.x_dev, xdt, pr.M, pr.K, pr.packed_dev, pr.N, pr.y_dev,
                                    nullptr, nullptr, nullptr);
        if (rc != BITLINEAR_OK)
            return rc;
        if (pr.M == 0)
            continue;
        const int64_t xrow = b3 ? (pr.K + 159) / 160 * 160 : pr.K;
        if (!gemv_fits(pr.M, xrow))
            return BITLINEAR_ERR_SHAPE;
        max_M = std::max(max_M, pr.M);
        max_xq = std::max(max_xq, pr.M * xrow);
        jobs[*n] = GemvJob{pr.x_dev,      static_cast<int>(pr.M), static_cast<int>(pr.K),
                           static_cast<int>(pr.N), pr.packed_dev, pr.gamma, pr.y_dev,
                           nullptr, nullptr, nullptr, nullptr, 0.0f};
        jobs[(*n)++].b3 = b3;
    }
    // one launch holds the largest x~ next to the largest problem's token tile
    if (*n > 0 && max_xq > gemv_max_xq(max_M))
        return BITLINEAR_ERR_SHAPE;
    return BITLINEAR_OK;
}

// Copies `count` pieces of sizes[i] bytes between one packed host buffer and
// the device pointers dev[i], merging pieces that lie back to back on the
// device into one copy.
int copy_pieces(const void *const *dev, const size_t *sizes, int count, char *host,
                cudaMemcpyKind kind, cudaStream_t st)
{
    int i = 0;
    while (i < count) {
        char *start = static_cast<char *>(const_cast<void *>(dev[i]));
        size_t bytes = sizes[i];
        int j = i + 1;
        while (j < count && static_cast<const char *>(dev[j]) == start + bytes) {
            bytes += sizes[j];
            ++j;
        }
        if (bytes > 0) {
            cudaError_t e = kind == cudaMemcpyHostToDevice
                                ? cudaMemcpyAsync(start, host, bytes, kind, st)
                                : cudaMemcpyAsync(host, start, bytes, kind, st);
            if (e != cudaSuccess)
                return BITLINEAR_ERR_CUDA;
        }
        host += bytes;
        i = j;
    }
    return BITLINEAR_OK;
}

}  // namespace

extern "C" int bitlinear_forward_grouped(const bitlinear_problem *problems, int count,
                                         bitlinear_dtype xdt, void *cuda_stream)
{
    GemvJob jobs[gemv::MAX_PROBLEMS];
    int n = 0;
    int rc = collect_gemv_group(problems, count, xdt, jobs, &n);
    if (rc != BITLINEAR_OK || n == 0)
        return rc;
    DeviceInfo *dev = nullptr;
    rc = current_device(&dev);
    if (rc != BITLINEAR_OK)
        return rc;
    return launch_gemv(jobs, n, xdt, *dev, static_cast<cudaStream_t>(cuda_stream));
}

// The device address of host memory the device can read and write (pinned
// and mapped into its address space), or null for any other pointer.
void *mapped_device_ptr(const void *host)
{
    cudaPointerAttributes a = {};
    if (cudaPointerGetAttributes(&a, host) != cudaSuccess) {
        cudaGetLastError();                       // not a pointer CUDA knows: clear it
        return nullptr;
    }
    return a.type == cudaMemoryTypeHost ? a.devicePointer : nullptr;
}

extern "C" int bitlinear_forward_grouped_b3(const bitlinear_problem *problems, int count,
                                            bitlinear_dtype xdt, void *cuda_stream)
{
    GemvJob jobs[gemv::MAX_PROBLEMS];
    int n = 0;
    int rc = collect_gemv_group(problems, count, xdt, jobs, &n, true);
    if (rc != BITLINEAR_OK || n == 0)
        return rc;
    DeviceInfo *dev = nullptr;
    rc = current_device(&dev);
    if (rc != BITLINEAR_OK)
        return rc;
    return launch_gemv(jobs, n, xdt, *dev, static_cast<cudaStream_t>(cuda_stream));
}

extern "C" int bitlinear_forward_grouped_host(const bitlinear_problem *problems, int count,
                                              bitlinear_dtype xdt, const void *x_host,
                                              void *y_host, void *cuda_stream)
{
    GemvJob jobs[gemv::MAX_PROBLEMS];
    int n = 0;
    int rc = collect_gemv_group(problems, count, xdt, jobs, &n);
    if (rc != BITLINEAR_OK)
        return rc;
    if (x_host == nullptr || y_host == nullptr)
        return BITLINEAR_ERR_ARG;
    if (n == 0)
        return BITLINEAR_OK;
    DeviceInfo *dev = nullptr;
    rc = current_device(&dev);
    if (rc != BITLINEAR_OK)
        return rc;
    const size_t xsize = xdt == BITLINEAR_BF16 ? 2 : 4;
    const void *xd[gemv::MAX_PROBLEMS];
    const void *yd[gemv::MAX_PROBLEMS];
    size_t xb[gemv::MAX_PROBLEMS], yb[gemv::MAX_PROBLEMS];
    size_t x_total = 0;
    for (int i = 0; i < n; ++i) {
        xd[i] = jobs[i].x;
        xb[i] = size_t(jobs[i].M) * jobs[i].K * xsize;     // a multiple of 256 (K % 128 == 0)
        yd[i] = jobs[i].y;
        yb[i] = size_t(jobs[i].M) * jobs[i].N * 2;
        x_total += xb[i];
    }
    cudaStream_t st = static_cast<cudaStream_t>(cuda_stream);

    // Tokens: host memory the device can read is staged by a kernel (no
    // copy-engine transfer); any other host memory by cudaMemcpyAsync.
    const void *x_map = mapped_device_ptr(x_host);
    if (x_map != nullptr && aligned(x_map, 16) && x_total / 16 <= INT_MAX) {
        stage::Pieces pc = {};
        pc.src = static_cast<const uint4 *>(x_map);
        pc.count = n;
        size_t end = 0;
        for (int i = 0; i < n; ++i) {
            pc.dst[i] = static_cast<uint4 *>(const_cast<void *>(xd[i]));
            end += xb[i] / 16;
            pc.end[i] = static_cast<int>(end);
        }
        const int vecs = static_cast<int>(end);
        const int per_cta = stage::THREADS * stage::PER_THREAD;
        const int grid = std::max(1, std::min((vecs + per_cta - 1) / per_cta, dev->sms));
        if (launch(stage::stage_tokens_kernel, dim3(grid), dim3(stage::THREADS), 0, st, pc) !=
            cudaSuccess)
            return BITLINEAR_ERR_CUDA;
    } else {
        rc = copy_pieces(xd, xb, n, static_cast<char *>(const_cast<void *>(x_host)),
                         cudaMemcpyHostToDevice, st);
        if (rc != BITLINEAR_OK)
            return rc;
    }

    // Outputs: into host memory the device can write, straight from the GEMV's
    // epilogue when every problem's part of it is 16-byte aligned (y_dev is
    // then not written); otherwise into y_dev and back by cudaMemcpyAsync.
    char *y_map = static_cast<char *>(mapped_device_ptr(y_host));
    bool direct = y_map != nullptr;
    for (size_t off = 0, i = 0; direct && i < static_cast<size_t>(n); off += yb[i], ++i)
        direct = aligned(y_map + off, 16);
    if (direct) {
        size_t off = 0;
        for (int i = 0; i < n; ++i) {
            jobs[i].y = y_map + off;
            off += yb[i];
        }
    }
    rc = launch_gemv(jobs, n, xdt, *dev, st);
    if (rc != BITLINEAR_OK || direct)
        return rc;
    return copy_pieces(yd, yb, n, static_cast<char *>(y_host), cudaMemcpyDeviceToHost, st);
}

namespace {

// Checks a problem list for the grouped calls and collects the non-empty
// problems. Sets *all_gemv when every one of them fits the GEMV path at the
// automatic threshold.
int collect_group(const bitlinear_problem *problems, int count, int xdt, TcJob *jobs, int *n,
                  bool *all_gemv, bool shapes_only = false,
                  const float *const *gains = nullptr, float eps = 0.0f)
{
    if (problems == nullptr || count < 1 || count > wsg::MAX_PROBLEMS)
        return BITLINEAR_ERR_ARG;
    *n = 0;
    *all_gemv = true;
    int64_t max_M = 0, max_xq = 0;
    static const uint4 dummy = {};   // stands in for the pointers when sizing
    for (int i = 0; i < count; ++i) {
        const bitlinear_problem &pr = problems[i];
        int rc = shapes_only
                     ? check_forward_args(&dummy, xdt, pr.M, pr.K, &dummy, pr.N, &dummy, nullptr,
                                          nullptr, nullptr)
                     : check_forward_args(pr.x_dev, xdt, pr.M, pr.K, pr.packed_dev, pr.N,
                                          pr.y_dev, nullptr, nullptr, nullptr);
        if (rc != BITLINEAR_OK)
            return rc;
        if (pr.M == 0)
            continue;
        if (!(pr.M <= kAutoGemvMaxM && gemv_fits(pr.M, pr.K)))
            *all_gemv = false;
        max_M = std::max(max_M, pr.M);
        max_xq = std::max(max_xq, pr.M * pr.K);
        jobs[(*n)++] = TcJob{pr.x_dev,
                             static_cast<int>(pr.M),
                             static_cast<int>(pr.K),
                             static_cast<int>(pr.N),
                             pr.packed_dev,
                             pr.gamma,
                             pr.y_dev,
                             nullptr,
                             gains != nullptr ? gains[i] : nullptr,
                             eps};
    }
    // one GEMV launch holds the largest x~ next to the largest problem's token tile
    if (*n > 0 && max_xq > gemv_max_xq(max_M))
        *all_gemv = false;
    return BITLINEAR_OK;
}

}  // namespace

extern "C" size_t bitlinear_workspace_bytes_grouped(const bitlinear_problem *problems, int count)
{
    TcJob jobs[wsg::MAX_PROBLEMS];
    int n = 0;
    bool all_gemv = true;
    // The dtype does not change the size; BF16 only passes the argument check.
    if (collect_group(problems, count, BITLINEAR_BF16, jobs, &n, &all_gemv, true) != BITLINEAR_OK)
        return SIZE_MAX;
    if (n == 0 || all_gemv)
        return 0;
    return tc_group_bytes(jobs, n, true);
}

extern "C" int bitlinear_forward_grouped_ws(const bitlinear_problem *problems, int count,
                                            bitlinear_dtype xdt, void *workspace_dev,
                                            size_t workspace_bytes, void *cuda_stream)
{
    TcJob jobs[wsg::MAX_PROBLEMS];
    int n = 0;
    bool all_gemv = true;
    int rc = collect_group(problems, count, xdt, jobs, &n, &all_gemv);
    if (rc != BITLINEAR_OK)
        return rc;
    if (n == 0)
        return BITLINEAR_OK;
    DeviceInfo *dev = nullptr;
    rc = current_device(&dev);
    if (rc != BITLINEAR_OK)
        return rc;
    cudaStream_t st = static_cast<cudaStream_t>(cuda_stream);
    if (all_gemv) {
        GemvJob g[wsg::MAX_PROBLEMS];
        for (int i = 0; i < n; ++i)
            g[i] = GemvJob{jobs[i].x,     jobs[i].M, jobs[i].K, jobs[i].N, jobs[i].packed,
                           jobs[i].gamma, jobs[i].y, nullptr,   nullptr,   nullptr,
                           nullptr,       0.0f};
        return launch_gemv(g, n, xdt, *dev, st);
    }
    return run_tc_group(jobs, n, xdt, workspace_dev, workspace_bytes, nullptr, nullptr, *dev, st,
                        0, true);
}

extern "C" int bitlinear_forward_grouped_rmsnorm(const bitlinear_problem *problems,
                                                 const float *const *norm_gains_dev, int count,
                                                 float norm_eps, bitlinear_dtype xdt,
                                                 void *workspace_dev, size_t workspace_bytes,
                                                 void *cuda_stream)
{
    if (problems == nullptr || norm_gains_dev == nullptr || count < 1 ||
        count > wsg::MAX_PROBLEMS)
        return BITLINEAR_ERR_ARG;
    if (!(norm_eps > 0.0f) || !(norm_eps <= FLT_MAX))
        return BITLINEAR_ERR_ARG;
    for (int i = 0; i < count; ++i) {
        if (problems[i].M > 0 && norm_gains_dev[i] == nullptr)
            return BITLINEAR_ERR_ARG;
        if (!aligned(norm_gains_dev[i], 16))
            return BITLINEAR_ERR_ALIGN;
    }
    TcJob jobs[wsg::MAX_PROBLEMS];
    int n = 0;
    bool all_gemv = true;
    int rc = collect_group(problems, count, xdt, jobs, &n, &all_gemv, false, norm_gains_dev,
                           norm_eps);
    if (rc != BITLINEAR_OK)
        return rc;
    if (n == 0)
        return BITLINEAR_OK;
    DeviceInfo *dev = nullptr;
    rc = current_device(&dev);
    if (rc != BITLINEAR_OK)
        return rc;
    cudaStream_t st = static_cast<cudaStream_t>(cuda_stream);
    if (all_gemv) {
        GemvJob g[wsg::MAX_PROBLEMS];
        for (int i = 0; i < n; ++i)
            g[i] = GemvJob{jobs[i].x,     jobs[i].M, jobs[i].K, jobs[i].N, jobs[i].packed,
                           jobs[i].gamma, jobs[i].y, nullptr,   nullptr,   nullptr,
                           jobs[i].norm_gain, jobs[i].norm_eps};
        return launch_gemv(g, n, xdt, *dev, st);
    }
    return run_tc_group(jobs, n, xdt, workspace_dev, workspace_bytes, nullptr, nullptr, *dev, st,
                        0, true);
}

extern "C" int bitlinear_forward_inject_timeout(const void *x_dev, bitlinear_dtype xdt, int64_t M,
                                                int64_t K, const void *packed_dev, float gamma,
                                                int64_t N, void *y_dev, void *workspace_dev,
                                                size_t workspace_bytes, void *cuda_stream,
                                                int path, int timeout_us)
{
    if (timeout_us < 1 || timeout_us > 10 * 1000 * 1000)
        return BITLINEAR_ERR_ARG;
    if (path != BITLINEAR_PATH_GEMV && path != BITLINEAR_PATH_TC)
        return BITLINEAR_ERR_ARG;
    return forward_impl(x_dev, xdt, M, K, packed_dev, gamma, N, y_dev, workspace_dev,
                        workspace_bytes, cuda_stream, nullptr, nullptr, nullptr, path,
                        timeout_us);
}

extern "C" int bitlinear_get_fault(int *fault_out, void *cuda_stream)
{
    if (fault_out == nullptr)
        return BITLINEAR_ERR_ARG;
    if (cudaStreamSynchronize(static_cast<cudaStream_t>(cuda_stream)) != cudaSuccess)
        return BITLINEAR_ERR_CUDA;
    unsigned int word = 0;
    if (cudaMemcpyFromSymbol(&word, g_fault_word, sizeof(word)) != cudaSuccess)
        return BITLINEAR_ERR_CUDA;
    *fault_out = static_cast<int>(word);
    if (word != 0) {
        const unsigned int zero = 0;
        if (cudaMemcpyToSymbol(g_fault_word, &zero, sizeof(zero)) != cudaSuccess)
            return BITLINEAR_ERR_CUDA;
        return BITLINEAR_ERR_TIMEOUT;
    }
    return BITLINEAR_OK;
}

// ======================================================== no-allocation path
//
// For callers that cannot allocate device memory: the tensor-core path's
// scratch (x~, beta, row sums of x~) lives in this fixed-size array, which
// every GPU that loads the library holds until the process exits. Host code
// must not use the array's name as a device address; its address is looked
// up once per device with cudaGetSymbolAddress and handed to the kernels.

static __device__ __align__(256) unsigned char g_static_scratch[BITLINEAR_STATIC_SCRATCH_BYTES];

namespace {

std::mutex g_static_scratch_mutex;
void *g_static_scratch_ptr[kMaxDevices];

// Device address of g_static_scratch on device `dev` (which must be current).
int static_scratch_address(int dev, void **out)
{
    std::lock_guard<std::mutex> lock(g_static_scratch_mutex);
    if (g_static_scratch_ptr[dev] == nullptr) {
        void *p = nullptr;
        if (cudaGetSymbolAddress(&p, g_static_scratch) != cudaSuccess || p == nullptr) {
            cudaGetLastError();
            return BITLINEAR_ERR_CUDA;
        }
        g_static_scratch_ptr[dev] = p;
    }
    *out = g_static_scratch_ptr[dev];
    return BITLINEAR_OK;
}

}  // namespace

extern "C" int bitlinear_forward_noalloc(const void *x_dev, bitlinear_dtype xdt, int64_t M,
                                         int64_t K, const void *packed_dev, float gamma,
                                         int64_t N, void *y_dev, void *cuda_stream)
{
    int rc = check_forward_args(x_dev, xdt, M, K, packed_dev, N, y_dev, nullptr, nullptr,
                                nullptr);
    if (rc != BITLINEAR_OK)
        return rc;
    if (M == 0)
        return BITLINEAR_OK;
    if (tc_base_bytes(M, K) > BITLINEAR_STATIC_SCRATCH_BYTES)
        return BITLINEAR_ERR_SCRATCH_LIMIT;
    DeviceInfo *dev = nullptr;
    rc = current_device(&dev);
    if (rc != BITLINEAR_OK)
        return rc;
    void *scratch = nullptr;
    rc = static_scratch_address(dev->id, &scratch);
    if (rc != BITLINEAR_OK)
        return rc;
    return run_tc_path(x_dev, xdt, static_cast<int>(M), static_cast<int>(K), packed_dev, gamma,
                       static_cast<int>(N), y_dev, scratch, BITLINEAR_STATIC_SCRATCH_BYTES,
                       nullptr, nullptr, nullptr, *dev, static_cast<cudaStream_t>(cuda_stream),
                       0, false);
}
