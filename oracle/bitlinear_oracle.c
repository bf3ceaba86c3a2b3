/*
 * bitlinear_oracle.c -- plain CPU statement of the BitNet b1.58 BitLinear
 * W1.58A8 matmul.
 *
 * TEST INFRASTRUCTURE. Only the tests, the smoke check and the CPU-baseline
 * leg of the benchmark may load or run this code. It shares nothing with the
 * CUDA library (no headers, no helpers, no tables) and the library never
 * calls it. It is written to be read against the pages, not to be fast:
 * single-threaded loops, fp32 where the pages' PyTorch listing computes in
 * fp32, a double accumulator for the weight mean.
 *
 * What it follows (page "BitNet b1.58 2B4T Guide: Scaling Native 1-Bit LLMs"):
 *   - section "Ternary Weight Quantization: absmean Scaling": gamma is the mean
 *     of |W| over the whole d_out x d_in matrix, and each weight becomes
 *     Clip(Round(W / gamma), -1, 1);
 *   - section "8-Bit Activation Quantization: absmax Scaling": per token,
 *     beta = max_j |x_j| and x~ = Clip(Round(x * Q_b / beta)), Q_b = 127;
 *   - section "Matrix Multiplication as Pure Integer Addition":
 *     y = (x~ W~^T) * beta * gamma / Q_b, the product being an integer sum;
 *   - the listing's RMSNorm ahead of the activation quantisation
 *     (oracle_rmsnorm, for the normalising forms of the path);
 *   - the gated ReLU^2 between the gate/up and down projections of the
 *     feed-forward block (oracle_relu2_glu, for the FFN chain);
 *   - the page's PyTorch listing (WeightQuantFunction.forward,
 *     quantize_activations_int8, BitLinear.forward), which fixes what the
 *     formulas leave open: the epsilon is a clamp(min=1e-5) of gamma and beta,
 *     Round is torch.round (ties to even), the activation scale is applied as
 *     x * (127 / beta), the activation clip range is [-128, 127] and the
 *     output scale is (beta * gamma) / 127.
 * Readings taken where the pages are silent (all listed in the design notes):
 *   - arithmetic is IEEE fp32 with round-to-nearest-even, bf16 inputs are
 *     widened to fp32 exactly, and the output is rounded once to bf16 (RNE);
 *   - the |W| sum is accumulated in double and divided once, then cast to fp32;
 *   - one gamma per weight matrix (the formula's double sum over i and j).
 *
 * The packed 2-bit layout (oracle_pack_codes) is the storage format the
 * library's packer must produce; it is written here from its specification
 * (see the layout comment above oracle_pack_codes), not from the library.
 *
 * Build: gcc -O2 -std=c11 -fPIC -shared -ffp-contract=off -fno-fast-math
 * (plus -fopenmp for the all-core copy that only the benchmark's CPU baseline
 * times: the integer products' independent outputs then run on all cores)
 */
#include <math.h>
#include <stdint.h>
#include <string.h>

/* clamp(min=1e-5) applied to gamma and beta in the page's listing */
static const float ORACLE_EPS = 1e-5f;
/* Q_b = 2^(b-1) with b = 8 bits, used as 127 by the page */
static const float ORACLE_QB = 127.0f;

/* ---------------------------------------------------------------- weights */

/* gamma = max(mean_{i,j} |W_ij|, 1e-5) over a row-major [N][K] fp32 matrix.
 * Section "Ternary Weight Quantization: absmean Scaling" (the double sum over
 * d_out and d_in divided by d_out * d_in); the clamp is the listing's. */
float oracle_absmean_gamma(const float *W, int64_t N, int64_t K)
{
    const int64_t count = N * K;
    if (count <= 0)
        return ORACLE_EPS;
    double sum = 0.0;
    for (int64_t i = 0; i < count; ++i)
        sum += fabs((double)W[i]);
    float gamma = (float)(sum / (double)count);
    if (gamma < ORACLE_EPS)
        gamma = ORACLE_EPS;
    return gamma;
}

/* W~ = Clip(Round(W / gamma), -1, 1) elementwise, Round = ties-to-even.
 * Same section; the fp32 division is the listing's weight / gamma. */
void oracle_ternarize(const float *W, int64_t N, int64_t K, float gamma,
                      int8_t *Wq)
{
    const int64_t count = N * K;
    for (int64_t i = 0; i < count; ++i) {
        float q = rintf(W[i] / gamma);
        if (q > 1.0f)
            q = 1.0f;
        if (q < -1.0f)
            q = -1.0f;
        Wq[i] = (int8_t)q;
    }
}

/* ------------------------------------------------------------ activations */

/* Exact widening of bf16 bit patterns to fp32 (bf16 is the top half of an
 * IEEE single). */
void oracle_bf16_to_f32(const uint16_t *in, int64_t n, float *out)
{
    for (int64_t i = 0; i < n; ++i) {
        uint32_t bits = (uint32_t)in[i] << 16;
        memcpy(&out[i], &bits, sizeof(float));
    }
}

/* RMS normalisation of each token row of a row-major [M][K] fp32 matrix,
 * before its quantisation: the RMSNorm member of the page's BitLinear listing
 * (step 1 of BitLinear.forward, torch's nn.RMSNorm over in_features), which
 * the bako.co page's forward flow also puts first ("the input activations
 * are normalized", section "Architecting the 1-Bit Paradigm").
 *   out_mk = (x_mk * r_m) * g_k,  r_m = 1 / sqrt(mean_k x_mk^2 + eps)
 * with g [K] the learned per-channel gain (ones at initialisation).
 * Readings where the pages are silent: the sum of squares is accumulated in
 * double (each fp32 square is exact there) and the mean is rounded once to
 * fp32; sqrt and the division are IEEE fp32, correctly rounded; eps is the
 * caller's (nn.RMSNorm's default is the machine epsilon of the compute type,
 * 2^-23 for fp32). */
void oracle_rmsnorm(const float *x, int64_t M, int64_t K, const float *g,
                    float eps, float *out)
{
    for (int64_t m = 0; m < M; ++m) {
        const float *row = x + m * K;
        double ss = 0.0;
        for (int64_t k = 0; k < K; ++k) {
            const double v = (double)row[k];
            ss += v * v;
        }
        const float ms = (float)(ss / (double)K);
        const float r = 1.0f / sqrtf(ms + eps);
        for (int64_t k = 0; k < K; ++k)
            out[m * K + k] = (row[k] * r) * g[k];
    }
}

/* Per-token absmax int8 quantisation of a row-major [M][K] fp32 matrix.
 * beta_m = max(max_k |x_mk|, 1e-5); x~_mk = Clip(Round(x_mk * (127 / beta_m)),
 * -128, 127). Section "8-Bit Activation Quantization: absmax Scaling" and the
 * listing's quantize_activations_int8. */
void oracle_quant_act(const float *x, int64_t M, int64_t K, int8_t *xq,
                      float *beta)
{
    for (int64_t m = 0; m < M; ++m) {
        const float *row = x + m * K;
        float b = 0.0f;
        for (int64_t k = 0; k < K; ++k) {
            float a = fabsf(row[k]);
            if (a > b)
                b = a;
        }
        if (b < ORACLE_EPS)
            b = ORACLE_EPS;
        const float scale = ORACLE_QB / b;
        for (int64_t k = 0; k < K; ++k) {
            float q = rintf(row[k] * scale);
            if (q > 127.0f)
                q = 127.0f;
            if (q < -128.0f)
                q = -128.0f;
            xq[m * K + k] = (int8_t)q;
        }
        beta[m] = b;
    }
}

/* ------------------------------------------------------- integer product */

/* acc_mn = sum_k x~_mk * W~_nk with x~ [M][K] and W~ [N][K], both row-major.
 * Section "Matrix Multiplication as Pure Integer Addition": the contraction
 * over d_in with W stored d_out x d_in, i.e. y = x W^T. */
void oracle_matmul_i32(const int8_t *xq, const int8_t *Wq, int64_t M,
                       int64_t N, int64_t K, int32_t *acc)
{
    /* Built with -fopenmp (the all-core CPU baseline only), the independent
     * outputs are shared between threads; each is still the same plain sum. */
#ifdef _OPENMP
#pragma omp parallel for collapse(2) schedule(static)
#endif
    for (int64_t m = 0; m < M; ++m) {
        for (int64_t n = 0; n < N; ++n) {
            int64_t s = 0;
            for (int64_t k = 0; k < K; ++k)
                s += (int64_t)xq[m * K + k] * (int64_t)Wq[n * K + k];
            acc[m * N + n] = (int32_t)s;
        }
    }
}

/* The same sum for a list of (m, n) pairs only, so that large shapes can be
 * checked on sampled outputs. */
void oracle_matmul_i32_pairs(const int8_t *xq, const int8_t *Wq, int64_t K,
                             const int64_t *ms, const int64_t *ns,
                             int64_t count, int32_t *acc)
{
#ifdef _OPENMP
#pragma omp parallel for schedule(static)
#endif
    for (int64_t i = 0; i < count; ++i) {
        const int8_t *a = xq + ms[i] * K;
        const int8_t *w = Wq + ns[i] * K;
        int64_t s = 0;
        for (int64_t k = 0; k < K; ++k)
            s += (int64_t)a[k] * (int64_t)w[k];
        acc[i] = (int32_t)s;
    }
}

/* ----------------------------------------------------------------- rescale */

/* fp32 -> bf16 with round-to-nearest, ties to even, on the bit pattern:
 * keep the upper 16 bits and look at the 16 discarded ones. More than half an
 * ulp rounds up, exactly half rounds to the even kept value. A carry out of
 * the mantissa bumps the exponent, which is the correct rounded result and
 * turns the largest finite values into infinity when they round past it.
 * NaN stays NaN (quiet bit forced). */
uint16_t oracle_f32_to_bf16(float f)
{
    uint32_t u;
    memcpy(&u, &f, sizeof(u));
    if ((u & 0x7f800000u) == 0x7f800000u && (u & 0x007fffffu) != 0u)
        return (uint16_t)((u >> 16) | 0x0040u);
    uint32_t kept = u >> 16;
    uint32_t dropped = u & 0xffffu;
    if (dropped > 0x8000u || (dropped == 0x8000u && (kept & 1u)))
        kept += 1u;
    return (uint16_t)kept;
}

void oracle_f32_to_bf16_array(const float *in, int64_t n, uint16_t *out)
{
    for (int64_t i = 0; i < n; ++i)
        out[i] = oracle_f32_to_bf16(in[i]);
}

/* y_mn = bf16( float(acc_mn) * ((beta_m * gamma) / 127) ), fp32 arithmetic.
 * Section "Matrix Multiplication as Pure Integer Addition" (rescale by
 * beta * gamma / Q_b) and the listing's BitLinear.forward step 5. */
void oracle_rescale_bf16(const int32_t *acc, const float *beta, float gamma,
                         int64_t M, int64_t N, uint16_t *y)
{
    for (int64_t m = 0; m < M; ++m) {
        const float s = (beta[m] * gamma) / ORACLE_QB;
        for (int64_t n = 0; n < N; ++n)
            y[m * N + n] = oracle_f32_to_bf16((float)acc[m * N + n] * s);
    }
}

/* -------------------------------------------------------------- FFN chain */

/* Gated squared-ReLU of the feed-forward block, elementwise over n values:
 *   h_i = (r_i * r_i) * up_i,  r_i = max(gate_i, 0)
 * The winbuzzer.com release article (section "Under the Hood") says ReLU^2
 * replaces SwiGLU in the model's feed-forward networks, and the bako.co page
 * names ReLU^2 as the FFN activation; replacing the Swish of SwiGLU keeps its
 * gate, so ReLU^2 applies to the gate projection's output and multiplies the
 * up projection's output elementwise. fp32 arithmetic in that order; when
 * gate and up hold bf16 values (the BitLinear outputs) every product is exact
 * in fp32 (at most 8 + 8 + 8 significant bits). A non-positive gate gives a
 * zero (of the sign of up). */
void oracle_relu2_glu(const float *gate, const float *up, int64_t n, float *h)
{
    for (int64_t i = 0; i < n; ++i) {
        const float r = gate[i] > 0.0f ? gate[i] : 0.0f;
        h[i] = (r * r) * up[i];
    }
}

/* ------------------------------------------------------------ 2-bit layout */

/* Packed ternary storage (the "2-bit nibbles" of the bitnet.xin guide, section
 * "Core Architecture"; the layout itself is this library's own):
 *   - rows are taken in blocks of 16 consecutive rows; block b occupies the
 *     16 * K / 4 bytes starting at byte b * 16 * K / 4, and when N is not a
 *     multiple of 16 the last block is completed with rows of zero weights;
 *   - inside a block the weights come in k-groups of 128: group g (the
 *     weights k in [128g, 128g + 128) of all 16 rows) occupies the 512 bytes at
 *     offset 512 g, and row r of the block the 32 bytes at offset 32 r in it;
 *   - those 32 bytes are 8 little-endian 32-bit words; word w holds the 16
 *     weights k = 128g + 16w + 4j + b (j, b in 0..3) in bits 8b + 2j and
 *     8b + 2j + 1, as the code W~ + 1 (0, 1 or 2).
 * The output holds ceil(N / 16) * 16 * K / 4 bytes. Returns 0, or -1 when K
 * is not a positive multiple of 128 or a weight is not ternary. */
int oracle_pack_codes(const int8_t *Wq, int64_t N, int64_t K, uint8_t *packed)
{
    if (K <= 0 || K % 128 != 0)
        return -1;
    const int64_t blocks = (N + 15) / 16;
    const int64_t row_bytes = K / 4;
    for (int64_t blk = 0; blk < blocks; ++blk) {
        for (int64_t r = 0; r < 16; ++r) {
            const int64_t n = 16 * blk + r;
            for (int64_t g = 0; g < K / 128; ++g) {
                for (int64_t w = 0; w < 8; ++w) {
                    uint32_t word = 0;
                    for (int j = 0; j < 4; ++j) {
                        for (int b = 0; b < 4; ++b) {
                            const int64_t k = 128 * g + 16 * w + 4 * j + b;
                            const int v = (n < N) ? Wq[n * K + k] : 0;
                            if (v < -1 || v > 1)
                                return -1;
                            word |= (uint32_t)(v + 1) << (8 * b + 2 * j);
                        }
                    }
                    uint8_t *dst = packed + blk * 16 * row_bytes + 512 * g + 32 * r + 4 * w;
                    dst[0] = (uint8_t)(word & 0xffu);
                    dst[1] = (uint8_t)((word >> 8) & 0xffu);
                    dst[2] = (uint8_t)((word >> 16) & 0xffu);
                    dst[3] = (uint8_t)((word >> 24) & 0xffu);
                }
            }
        }
    }
    return 0;
}

/* ------------------------------------------------- base-3 layout (5 per byte) */

/* Denser storage of the same codes, 5 per byte (3^5 = 243 <= 256, 1.6 bits
 * per weight): the log2(3) = 1.58-bit density behind the 0.4 GB footprint
 * of the 2B model ("Microsoft Releases BitNet b1.58 2B4T", opening section;
 * "BitNet b1.58 2B4T Guide", section "Mathematical Architecture"). The layout
 * is this library's own:
 *   - K is padded with zero weights to Kp, a multiple of 160; rows come in
 *     blocks of 16 (the last block completed with zero rows); block b
 *     occupies the 16 * Kp / 5 bytes starting at byte b * 16 * Kp / 5;
 *   - inside a block the weights come in k-groups of 160: group g holds the
 *     weights k in [160 g, 160 g + 160) of all 16 rows in the 512 bytes at
 *     offset 512 g, row r of the block in the 32 bytes at offset 32 r;
 *   - those 32 bytes hold the 160 codes c = W~ + 1 of the row in "stream
 *     order": stream position p = 16 w + 4 b + j is the weight
 *     k = 160 g + 16 w + 4 j + b (w in 0..9, j, b in 0..3) -- the order of the
 *     2-bit fields of the 2-bit layout's words, read from bit 0 up;
 *   - byte B (0..31) holds the codes of stream positions 5 B .. 5 B + 4 as
 *     the number sum_i c(5 B + i) * 3^i (0..242).
 * The output holds ceil(N / 16) * 16 * Kp / 5 bytes. Returns 0, or -1 when K
 * is not a positive multiple of 128 or a weight is not ternary. */
int oracle_pack_codes_b3(const int8_t *Wq, int64_t N, int64_t K, uint8_t *packed)
{
    if (K <= 0 || K % 128 != 0)
        return -1;
    const int64_t Kp = (K + 159) / 160 * 160;
    const int64_t blocks = (N + 15) / 16;
    const int64_t row_bytes = Kp / 5;
    for (int64_t blk = 0; blk < blocks; ++blk) {
        for (int64_t r = 0; r < 16; ++r) {
            const int64_t n = 16 * blk + r;
            for (int64_t g = 0; g < Kp / 160; ++g) {
                for (int64_t B = 0; B < 32; ++B) {
                    int value = 0;
                    int power = 1;
                    for (int i = 0; i < 5; ++i) {
                        const int64_t p = 5 * B + i;          /* stream position */
                        const int64_t w = p / 16, b = (p % 16) / 4, j = p % 4;
                        const int64_t k = 160 * g + 16 * w + 4 * j + b;
                        const int v = (n < N && k < K) ? Wq[n * K + k] : 0;
                        if (v < -1 || v > 1)
                            return -1;
                        value += (v + 1) * power;
                        power *= 3;
                    }
                    packed[blk * 16 * row_bytes + 512 * g + 32 * r + B] = (uint8_t)value;
                }
            }
        }
    }
    return 0;
}
