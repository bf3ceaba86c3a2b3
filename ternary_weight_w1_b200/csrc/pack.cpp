// Offline absmean ternarisation and packing of BitLinear weights (host): the
// 2-bit layout, and the denser base-3 layout (five codes per byte).
//
// Page "BitNet b1.58 2B4T Guide: Scaling Native 1-Bit LLMs", section "Ternary
// Weight Quantization: absmean Scaling": gamma is the mean of |W| over the
// whole d_out x d_in matrix and each weight becomes Clip(Round(W / gamma), -1,
// 1); the page's listing (WeightQuantFunction.forward) clamps gamma at 1e-5,
// divides in the weight dtype (fp32 here) and rounds half to even. The codes
// are stored two bits each in the layout documented in include/bitlinear.h.
//
// The mean is accumulated in double over fixed 1 Mi-element blocks whose sums
// are added in block order, so gamma does not depend on the thread count.
// Must be compiled without fast-math (IEEE division and rounding).

#include <algorithm>
#include <climits>
#include <cmath>
#include <cstdint>
#include <cstring>
#include <thread>
#include <vector>

#include "../../include/bitlinear.h"

namespace {

constexpr float kEps = 1e-5f;
constexpr int64_t kBlock = int64_t(1) << 20;

unsigned worker_count(int64_t work_items)
{
    unsigned hw = std::thread::hardware_concurrency();
    if (hw == 0)
        hw = 1;
    hw = std::min(hw, 32u);
    int64_t useful = std::max<int64_t>(1, work_items);
    return static_cast<unsigned>(std::min<int64_t>(hw, useful));
}

// Runs fn(0 .. count-1) over worker threads (fn must be safe to call
// concurrently for different i). If a thread cannot be created, the items not
// yet handed out run on the calling thread instead.
template <class Fn>
void parallel_for(int64_t count, Fn fn)
{
    const unsigned workers = worker_count(count);
    std::vector<std::thread> pool;
    int64_t handed_out = 0;
    if (workers > 1) {
        try {
            pool.reserve(workers);
            for (unsigned t = 0; t < workers; ++t) {
                const int64_t lo = count * t / workers;
                const int64_t hi = count * (t + 1) / workers;
                pool.emplace_back([=, &fn] {
                    for (int64_t i = lo; i < hi; ++i)
                        fn(i);
                });
                handed_out = hi;
            }
        } catch (...) {
        }
    }
    for (int64_t i = handed_out; i < count; ++i)
        fn(i);
    for (auto &th : pool)
        th.join();
}

// Ternary code (W~ + 1) of one latent weight.
inline uint32_t ternary_code(float w, float gamma)
{
    float r = std::nearbyint(w / gamma);  // default rounding mode: ties to even
    if (r > 1.0f)
        r = 1.0f;
    else if (r < -1.0f)
        r = -1.0f;
    return static_cast<uint32_t>(static_cast<int>(r) + 1);
}

}  // namespace

extern "C" size_t bitlinear_packed_bytes(int64_t N, int64_t K)
{
    if (N < 1 || K < 128 || K % 128 != 0)
        return 0;
    const int64_t blocks = N / 16 + (N % 16 != 0 ? 1 : 0);
    if (K / 4 > INT64_MAX / 16 / blocks)          // the size would not fit in 64 bits
        return 0;
    return static_cast<size_t>(blocks) * 16 * static_cast<size_t>(K / 4);
}

namespace {

// gamma = max(mean |W|, 1e-5): double accumulation in fixed blocks, added in
// block order, then one cast.
float absmean_gamma(const float *W_host, int64_t N, int64_t K)
{
    const int64_t total = N * K;
    const int64_t blocks = (total + kBlock - 1) / kBlock;
    std::vector<double> partial(static_cast<size_t>(blocks), 0.0);
    parallel_for(blocks, [&](int64_t b) {
        const int64_t lo = b * kBlock;
        const int64_t hi = std::min(total, lo + kBlock);
        double s = 0.0;
        for (int64_t i = lo; i < hi; ++i)
            s += std::fabs(static_cast<double>(W_host[i]));
        partial[static_cast<size_t>(b)] = s;
    });
    double sum = 0.0;
    for (double s : partial)
        sum += s;
    float gamma = static_cast<float>(sum / static_cast<double>(total));
    if (!(gamma >= kEps))
        gamma = kEps;
    return gamma;
}

// One 2-bit-layout word: the 16 weights k0 .. k0 + 15 of row n, weight
// k0 + 4j + b at bits 8b + 2j as the code W~ + 1; weights past the row (or
// rows past N) are zeros (code 1).
inline uint32_t code_word(const float *W_host, int64_t N, int64_t K, int64_t n, int64_t k0,
                          float gamma)
{
    uint32_t word = 0;
    for (int k = 0; k < 16; ++k) {
        const uint32_t code = (n < N && k0 + k < K) ? ternary_code(W_host[n * K + k0 + k], gamma)
                                                    : 1u;
        word |= code << (8 * (k & 3) + 2 * (k >> 2));
    }
    return word;
}

int pack_weights(const float *W_host, int64_t N, int64_t K, void *packed_host, float *gamma_out)
{
    const float gamma = absmean_gamma(W_host, N, K);
    // Row blocks of 16 rows; inside a block, k-groups of 128 weights laid out
    // as 16 rows x 32 bytes; word w of a (row, group) holds
    // k = 128g + 16w + 4j + b at bit 8b + 2j. Rows past N are zero weights.
    uint8_t *out = static_cast<uint8_t *>(packed_host);
    const int64_t row_blocks = (N + 15) / 16;
    const int64_t groups = K / 128;
    const size_t block_bytes = 16 * static_cast<size_t>(K / 4);
    parallel_for(row_blocks * 16, [&](int64_t n) {
        const int64_t blk = n / 16;
        const int64_t r = n % 16;
        uint8_t *block = out + static_cast<size_t>(blk) * block_bytes;
        for (int64_t g = 0; g < groups; ++g) {
            uint8_t *dst = block + 512 * g + 32 * r;
            for (int w = 0; w < 8; ++w) {
                const uint32_t word = code_word(W_host, N, K, n, 128 * g + 16 * w, gamma);
                std::memcpy(dst + 4 * w, &word, 4);  // little-endian host
            }
        }
    });
    *gamma_out = gamma;
    return BITLINEAR_OK;
}

// The base-3 layout: K padded to Kp (a multiple of 160), k-groups of 160
// weights as 16 rows x 32 bytes. A (row, group)'s codes are the ten 2-bit
// layout words of its 160 weights read as one stream of 2-bit fields from bit
// 0 up; byte B holds stream fields 5B .. 5B + 4 as base-3 digits 0 .. 4.
int pack_weights_b3(const float *W_host, int64_t N, int64_t K, void *packed_host,
                    float *gamma_out)
{
    const float gamma = absmean_gamma(W_host, N, K);
    uint8_t *out = static_cast<uint8_t *>(packed_host);
    const int64_t Kp = (K + 159) / 160 * 160;
    const int64_t row_blocks = (N + 15) / 16;
    const int64_t groups = Kp / 160;
    const size_t block_bytes = 16 * static_cast<size_t>(Kp / 5);
    parallel_for(row_blocks * 16, [&](int64_t n) {
        const int64_t blk = n / 16;
        const int64_t r = n % 16;
        uint8_t *block = out + static_cast<size_t>(blk) * block_bytes;
        for (int64_t g = 0; g < groups; ++g) {
            uint32_t words[10];
            for (int w = 0; w < 10; ++w)
                words[w] = code_word(W_host, N, K, n, 160 * g + 16 * w, gamma);
            uint8_t *dst = block + 512 * g + 32 * r;
            for (int B = 0; B < 32; ++B) {
                uint32_t value = 0;
                for (int i = 4; i >= 0; --i) {            // Horner: digit 4 first
                    const int f = 5 * B + i;
                    value = 3 * value + ((words[f >> 4] >> (2 * (f & 15))) & 3u);
                }
                dst[B] = static_cast<uint8_t>(value);
            }
        }
    });
    *gamma_out = gamma;
    return BITLINEAR_OK;
}

}  // namespace

extern "C" int bitlinear_pack_weights(const float *W_host, int64_t N, int64_t K,
                                      void *packed_host, float *gamma_out)
{
    if (!W_host || !packed_host || !gamma_out || N < 1 || K < 0)
        return BITLINEAR_ERR_ARG;
    if (K < 128 || K % 128 != 0)
        return BITLINEAR_ERR_SHAPE;
    try {
        return pack_weights(W_host, N, K, packed_host, gamma_out);
    } catch (...) {
        // nothing crosses the C ABI; only host allocation can fail here
        return BITLINEAR_ERR_HOST;
    }
}

extern "C" size_t bitlinear_packed_bytes_b3(int64_t N, int64_t K)
{
    if (N < 1 || K < 128 || K % 128 != 0 || K > (int64_t(1) << 40))
        return 0;
    const int64_t blocks = N / 16 + (N % 16 != 0 ? 1 : 0);
    const int64_t row = (K + 159) / 160 * 32;      // bytes of one row: Kp / 5
    if (row > INT64_MAX / 16 / blocks)             // the size would not fit in 64 bits
        return 0;
    return static_cast<size_t>(blocks) * 16 * static_cast<size_t>(row);
}

extern "C" int bitlinear_pack_weights_b3(const float *W_host, int64_t N, int64_t K,
                                         void *packed_host, float *gamma_out)
{
    if (!W_host || !packed_host || !gamma_out || N < 1 || K < 0)
        return BITLINEAR_ERR_ARG;
    if (K < 128 || K % 128 != 0)
        return BITLINEAR_ERR_SHAPE;
    try {
        return pack_weights_b3(W_host, N, K, packed_host, gamma_out);
    } catch (...) {
        return BITLINEAR_ERR_HOST;
    }
}
