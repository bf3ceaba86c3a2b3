/*
 * bitlinear.h -- C ABI of libbitlinear, the BitNet b1.58 BitLinear W1.58A8
 * matmul for NVIDIA B200 (sm_100a).
 *
 * The operator (page "BitNet b1.58 2B4T Guide: Scaling Native 1-Bit LLMs"):
 *   - weights W in R^{d_out x d_in} are ternarised once by absmean scaling,
 *       gamma = max(mean_{i,j} |W_ij|, 1e-5),  W~ = Clip(Round(W / gamma), -1, 1)
 *     (section "Ternary Weight Quantization: absmean Scaling");
 *   - each token x in R^{d_in} is quantised to int8 by absmax scaling,
 *       beta = max(max_j |x_j|, 1e-5),  x~ = Clip(Round(x * (127 / beta)), -128, 127)
 *     (section "8-Bit Activation Quantization: absmax Scaling");
 *   - the product is an integer sum, rescaled once:
 *       y = bf16( float(x~ W~^T) * ((beta * gamma) / 127) )
 *     (section "Matrix Multiplication as Pure Integer Addition").
 * Round is round-half-to-even (torch.round in the page's PyTorch listing),
 * all floating point is IEEE fp32, and the output is rounded once to bf16.
 *
 * Notation: M tokens, K = d_in, N = d_out. x is [M][K] row-major, W is [N][K]
 * row-major, y is [M][N] row-major (y = x W^T).
 *
 * Conventions shared by every call:
 *   - Ownership: the caller allocates and frees every buffer. The library
 *     never allocates or frees memory; device buffers (x, packed weights, y,
 *     workspace, debug outputs) are plain device pointers.
 *   - Streams: cuda_stream is a cudaStream_t (NULL = the legacy default
 *     stream). All device work is enqueued asynchronously on it; nothing
 *     synchronises the host except bitlinear_get_fault.
 *   - Errors: every call returns a bitlinear_status; nothing throws across
 *     the ABI. Argument errors are detected on the host before any launch.
 *     BITLINEAR_ERR_CUDA reports a launch error (cudaGetLastError); faults of
 *     work already enqueued surface at the caller's next synchronisation.
 *   - Alignment: x, packed weights, y, workspace and int8 outputs must be
 *     16-byte aligned, fp32/int32 outputs 4-byte aligned.
 *   - Shapes: K must be a positive multiple of 128 for the device calls;
 *     M >= 0 (M = 0 is a no-op), N >= 1, K <= 65536 for the forward calls.
 *   - Values: activations are finite; a token holding a NaN has unspecified
 *     outputs (an infinity makes beta infinite, as in the page's listing).
 */
#ifndef BITLINEAR_H
#define BITLINEAR_H

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

#define BITLINEAR_ABI_VERSION 1

typedef enum {
    BITLINEAR_OK = 0,
    BITLINEAR_ERR_ARG = 1,       /* null pointer or negative size */
    BITLINEAR_ERR_SHAPE = 2,     /* K not a multiple of 128, a size out of range */
    BITLINEAR_ERR_ALIGN = 3,     /* a pointer misses its alignment */
    BITLINEAR_ERR_DTYPE = 4,     /* unknown bitlinear_dtype */
    BITLINEAR_ERR_CUDA = 5,      /* a CUDA runtime/driver call failed */
    BITLINEAR_ERR_TIMEOUT = 6,   /* a bounded device-side wait ran out */
    BITLINEAR_ERR_WORKSPACE = 7, /* workspace missing or smaller than required */
    BITLINEAR_ERR_SCRATCH_LIMIT = 8, /* problem too large for the library's static scratch */
    BITLINEAR_ERR_HOST = 9,      /* a host allocation failed */
    BITLINEAR_ERR_IO = 10,       /* a file could not be opened, written or renamed */
    BITLINEAR_ERR_FORMAT = 11    /* not a valid packed-weight file (header, size or checksum) */
} bitlinear_status;

typedef enum {
    BITLINEAR_BF16 = 0,          /* x holds bf16 values (widened exactly to fp32) */
    BITLINEAR_FP32 = 1           /* x holds fp32 values */
} bitlinear_dtype;

/* Kernel choice for bitlinear_forward_ex. */
typedef enum {
    BITLINEAR_PATH_AUTO = 0,     /* pick by M (what bitlinear_forward does) */
    BITLINEAR_PATH_GEMV = 1,     /* fused-quant dp4a GEMV, M <= 16 */
    BITLINEAR_PATH_TC = 2        /* quant kernel + tcgen05 kind::i8 GEMM */
} bitlinear_path;

/* ---------------------------------------------------------------- packing */

/* Bytes of the packed ternary matrix for N rows of K weights:
 * ceil(N / 16) * 16 * K / 4. Returns 0 when N < 1, K is not a positive
 * multiple of 128, or the size does not fit in 64 bits.
 *
 * Packed layout (this library's own; the "2-bit nibbles" of the bitnet.xin
 * guide, section "Core Architecture"):
 *   - rows are taken in blocks of 16 consecutive rows; block b occupies the
 *     16 * K / 4 bytes starting at byte b * 16 * K / 4 (when N % 16 != 0 the
 *     last block is completed with rows of zero weights);
 *   - inside a block the weights come in k-groups of 128: group g holds the
 *     weights k in [128g, 128g + 128) of all 16 rows in the 512 bytes at
 *     offset 512 g, row r of the block in the 32 bytes at offset 32 r;
 *   - those 32 bytes are 8 little-endian 32-bit words; word w holds the 16
 *     weights k = 128g + 16w + 4j + b (j, b in 0..3) in bits 8b + 2j and
 *     8b + 2j + 1 as the code W~ + 1 (0, 1 or 2; 3 is unused).
 *   So every 512-byte (block, group) piece is contiguous, a block's weights
 *   are one contiguous byte range, and (word >> 2j) & 0x03030303 holds the
 *   codes of k = 128g + 16w + 4j .. +3 in the order of an int32 word of int8
 *   activations. */
size_t bitlinear_packed_bytes(int64_t N, int64_t K);

/* Offline absmean ternarisation and packing, on the host (no device work).
 *   W_host      [in]  latent fp32 weights, [N][K] row-major, host memory
 *   N, K        [in]  d_out, d_in; K must be a positive multiple of 128
 *   packed_host [out] caller-allocated host buffer of bitlinear_packed_bytes(N, K)
 *                     bytes (copy it to the device before bitlinear_forward)
 *   gamma_out   [out] gamma = max(mean |W|, 1e-5), the sum taken in double
 * Follows section "Ternary Weight Quantization: absmean Scaling" and the
 * listing's WeightQuantFunction.forward (W / gamma in fp32, ties to even,
 * clip to [-1, 1]). Returns BITLINEAR_ERR_ARG for null pointers or N < 1,
 * BITLINEAR_ERR_SHAPE for a bad K, BITLINEAR_ERR_HOST if a host allocation
 * fails. Runs on several host threads (on the calling thread alone when no
 * thread can be created); the result does not depend on their number. */
int bitlinear_pack_weights(const float *W_host, int64_t N, int64_t K,
                           void *packed_host, float *gamma_out);

/* ------------------------------------------------------- base-3 packing */

/* Bytes of the base-3 packed matrix: ceil(N / 16) * 16 * Kp / 5 with Kp = K
 * rounded up to a multiple of 160 (1.6 bits per weight, 20% less than the
 * 2-bit layout). 0 for the shapes bitlinear_packed_bytes refuses.
 *
 * Base-3 layout (this library's own; log2(3) = 1.58 bits per weight is what
 * puts the 2B model's non-embedding weights near 0.4 GB: "Microsoft Releases
 * BitNet b1.58 2B4T", opening section):
 *   - K is padded with zero weights to Kp; rows come in blocks of 16 (the last
 *     completed with zero rows); block b occupies the 16 * Kp / 5 bytes
 *     starting at byte b * 16 * Kp / 5;
 *   - inside a block the weights come in k-groups of 160: group g holds the
 *     weights k in [160g, 160g + 160) of all 16 rows in the 512 bytes at
 *     offset 512 g, row r of the block in the 32 bytes at offset 32 r;
 *   - those 32 bytes hold the 160 codes W~ + 1 of the row in stream order:
 *     stream position p = 16w + 4b + j is the weight k = 160g + 16w + 4j + b
 *     (the 2-bit fields of the 2-bit layout's words, read from bit 0 up);
 *   - byte B holds stream positions 5B .. 5B + 4 as sum_i code(5B + i) * 3^i. */
size_t bitlinear_packed_bytes_b3(int64_t N, int64_t K);

/* bitlinear_pack_weights into the base-3 layout: the same gamma and codes,
 * five per byte. packed_host holds bitlinear_packed_bytes_b3(N, K) bytes.
 * Errors as for bitlinear_pack_weights. */
int bitlinear_pack_weights_b3(const float *W_host, int64_t N, int64_t K,
                              void *packed_host, float *gamma_out);

/* bitlinear_forward on base-3 packed weights (a footprint option: 20% fewer
 * weight bytes in HBM, decoded in the GEMV through a 256-entry table in
 * shared memory). The GEMV path only: M <= 16 and M * Kp <= 196608, else
 * BITLINEAR_ERR_SHAPE before any device work. Arguments and results as for
 * bitlinear_forward, with packed_b3_dev holding
 * bitlinear_packed_bytes_b3(N, K) bytes; no workspace. */
int bitlinear_forward_b3(const void *x_dev, bitlinear_dtype xdt, int64_t M,
                         int64_t K, const void *packed_b3_dev, float gamma,
                         int64_t N, void *y_dev, void *cuda_stream,
                         int32_t *acc_dev_or_null, int8_t *xq_dev_or_null,
                         float *beta_dev_or_null);

/* ------------------------------------------------------ packed-weight files */

/* The packer's output stored once and loaded at serving time (the ternary
 * weights are exported once after training: "BitNet b1.58 2B4T Guide",
 * section "High-Precision Master Weights"). A file is a 64-byte little-endian
 * header followed by the payload:
 *   0  "BITLIN58"   8  u32 version (1)   12 u32 layout (1 = the layout above)
 *   16 i64 N        24 i64 K             32 f32 gamma       36 u32 0
 *   40 u64 payload bytes (= bitlinear_packed_bytes(N, K))
 *   48 u64 FNV-1a 64-bit hash of the payload                56 u64 0
 *   64 payload (the packed bytes, as bitlinear_pack_weights wrote them)
 * All three calls are host-only and thread-safe for different paths. */

/* Writes a packed matrix and its gamma to `path` (through "<path>.tmp" and a
 * rename, so the final name never holds a partial file). Returns
 * BITLINEAR_ERR_ARG for null pointers or a gamma that is not finite and > 0,
 * BITLINEAR_ERR_SHAPE for a bad (N, K), BITLINEAR_ERR_IO when the file
 * cannot be written. */
int bitlinear_save_packed(const char *path, const void *packed_host, int64_t N,
                          int64_t K, float gamma);

/* Reads only the header of `path`: N, K and gamma, so the caller can size
 * the payload buffer (bitlinear_packed_bytes(N, K)). BITLINEAR_ERR_IO when
 * the file cannot be opened, BITLINEAR_ERR_FORMAT for a bad header. */
int bitlinear_read_packed_header(const char *path, int64_t *N_out,
                                 int64_t *K_out, float *gamma_out);

/* Reads `path` into the caller's host buffer of packed_bytes bytes (at least
 * the payload) and returns N, K and gamma. The payload hash is checked:
 * BITLINEAR_ERR_FORMAT for a bad header, a truncated or over-long file or a
 * hash mismatch; BITLINEAR_ERR_ARG when the buffer is too small;
 * BITLINEAR_ERR_IO when the file cannot be opened. The outputs are written
 * only on success. */
int bitlinear_load_packed(const char *path, void *packed_host,
                          size_t packed_bytes, int64_t *N_out, int64_t *K_out,
                          float *gamma_out);

/* ------------------------------------------------- activation quantisation */

/* Per-token absmax int8 quantisation on the device.
 *   x_dev   [in]  [M][K] activations of type xdt, device memory
 *   xq_dev  [out] [M][K] int8 x~, device memory (16-byte aligned)
 *   beta_dev[out] [M] fp32 beta (the clamped absmax of each token)
 * Section "8-Bit Activation Quantization: absmax Scaling" and the listing's
 * quantize_activations_int8. One kernel launch on cuda_stream. */
int bitlinear_quant_act(const void *x_dev, bitlinear_dtype xdt, int64_t M,
                        int64_t K, int8_t *xq_dev, float *beta_dev,
                        void *cuda_stream);

/* ---------------------------------------------------------------- forward */

/* Device workspace bytes bitlinear_forward needs for (M, N, K): 0 when the
 * GEMV path is taken (M <= 6 and M * K <= 196608), else room for x~ (M*K
 * bytes), beta, the
 * per-token sums of x~, and the tensor-core GEMM's inter-CTA region (flag
 * words and int32 partial sums of tiles whose k-range is split between
 * CTAs; at most 192 * 128 * 192 * 4 bytes). The flag words are cleared by
 * the call itself before its GEMM reads them, so the workspace needs no
 * initialisation, but two calls that may run at the same time (different
 * streams) must not share one. Returns SIZE_MAX for invalid shapes. */
size_t bitlinear_workspace_bytes(int64_t M, int64_t N, int64_t K);

/* y = BitLinear(x) with pre-packed ternary weights, on the device.
 *   x_dev       [in]  [M][K] activations of type xdt
 *   packed_dev  [in]  packed weights (layout above), bitlinear_packed_bytes(N, K)
 *                     bytes
 *   gamma       [in]  the gamma bitlinear_pack_weights returned
 *   y_dev       [out] [M][N] bf16 (uint16 bit patterns)
 *   workspace_dev, workspace_bytes
 *               [in]  scratch of at least bitlinear_workspace_bytes(M, N, K)
 *                     bytes (may be NULL when that is 0); its contents are
 *                     overwritten
 *   acc_dev_or_null  [out, optional] [M][N] int32 x~ W~^T before rescaling
 *   xq_dev_or_null   [out, optional] [M][K] int8 x~
 *   beta_dev_or_null [out, optional] [M] fp32 beta
 * The optional outputs exist so that tests can compare the integer stages
 * bit for bit; pass NULL in production. M <= 6 with M * K <= 196608 runs one
 * fused kernel (quantisation in the prologue, dp4a over the packed weights);
 * other shapes run the quantisation kernel and the tcgen05 int8 tensor-core
 * GEMM, whose
 * results do not depend on how its work is split between CTAs (the int32
 * partial sums are exact). */
int bitlinear_forward(const void *x_dev, bitlinear_dtype xdt, int64_t M,
                      int64_t K, const void *packed_dev, float gamma,
                      int64_t N, void *y_dev, void *workspace_dev,
                      size_t workspace_bytes, void *cuda_stream,
                      int32_t *acc_dev_or_null, int8_t *xq_dev_or_null,
                      float *beta_dev_or_null);

/* bitlinear_forward with an explicit kernel choice (bitlinear_path).
 * BITLINEAR_PATH_GEMV needs M <= 16 and the tokens' x~ (M * K bytes) within
 * the GEMV's shared-memory limit of 196608 bytes; otherwise it returns
 * BITLINEAR_ERR_SHAPE, before any device work. Beside a large x~ the GEMV
 * streams its weights in smaller stages. The workspace for BITLINEAR_PATH_TC is
 * bitlinear_workspace_bytes_path(M, N, K, BITLINEAR_PATH_TC). */
int bitlinear_forward_ex(const void *x_dev, bitlinear_dtype xdt, int64_t M,
                         int64_t K, const void *packed_dev, float gamma,
                         int64_t N, void *y_dev, void *workspace_dev,
                         size_t workspace_bytes, void *cuda_stream,
                         int32_t *acc_dev_or_null, int8_t *xq_dev_or_null,
                         float *beta_dev_or_null, int path);

/* y = BitLinear(RMSNorm(x)): the tokens are RMS-normalised before their
 * absmax quantisation, as the page's BitLinear listing does with its
 * nn.RMSNorm(in_features) member (step 1 of BitLinear.forward), fused into the
 * quantisation pass of either path (the GEMV prologue or the quantisation
 * kernel ahead of the tensor-core GEMM). Per token m:
 *   r_m = 1 / sqrt(mean_k x_mk^2 + norm_eps),  x'_mk = (x_mk * r_m) * g_k
 * and x' takes the place of x in bitlinear_forward. The sum of squares is
 * accumulated in double and the mean rounded once to fp32; the square root,
 * the division and both products are IEEE fp32.
 *   norm_gain_dev [in] [K] fp32 gains g, device memory, 16-byte aligned
 *                      (may be NULL only when M = 0)
 *   norm_eps      [in] finite and > 0 (nn.RMSNorm's default for fp32 is the
 *                      fp32 machine epsilon, 2^-23)
 *   path          [in] a bitlinear_path, as for bitlinear_forward_ex
 * Every other argument, the workspace size and the dispatch are those of
 * bitlinear_forward_ex; xq_dev_or_null and beta_dev_or_null return the
 * quantised normalised tokens and their beta. Returns BITLINEAR_ERR_ARG for a
 * missing gain or a bad eps, BITLINEAR_ERR_ALIGN for a misaligned gain. */
int bitlinear_forward_rmsnorm(const void *x_dev, bitlinear_dtype xdt, int64_t M,
                              int64_t K, const float *norm_gain_dev,
                              float norm_eps, const void *packed_dev,
                              float gamma, int64_t N, void *y_dev,
                              void *workspace_dev, size_t workspace_bytes,
                              void *cuda_stream, int32_t *acc_dev_or_null,
                              int8_t *xq_dev_or_null, float *beta_dev_or_null,
                              int path);

/* ----------------------------------------------------- feed-forward chain */

/* Device workspace bytes bitlinear_ffn_forward needs for M tokens, whatever
 * gains it is given. For decode batches (M <= 6 and 2 M K <= 196608) it is
 * that of the down projection (M tokens of F features to K), i.e.
 * bitlinear_workspace_bytes(M, K, F), 0 when that projection takes the
 * GEMV path. Otherwise the gate/up launches' scratch and their two bf16
 * outputs, or the down projection's scratch if larger. SIZE_MAX for shapes
 * bitlinear_ffn_forward refuses. */
size_t bitlinear_workspace_bytes_ffn(int64_t M, int64_t K, int64_t F);

/* The feed-forward block of a BitNet b1.58 decoder layer for M decode tokens:
 *   gate = BitLinear_gate(x), up = BitLinear_up(x)        ([M][F], bf16)
 *   h    = (r * r) * up,  r = max(gate, 0)                 ([M][F], fp32)
 *   y    = BitLinear_down(h)                               ([M][K], bf16)
 * ReLU^2 replaces SwiGLU in the model's feed-forward networks ("Microsoft
 * Releases BitNet b1.58 2B4T", section "Under the Hood"; "BitNet b1.58: The
 * 1-Bit Paradigm Shift"), read here as gated: the squared ReLU of the gate
 * projection multiplies the up projection elementwise. h is computed in
 * fp32 from the two bf16 outputs (exact: every product of bf16 values fits
 * fp32). Each BitLinear is the one of bitlinear_forward (its own gamma); with
 * gains, each RMS-normalises its input first as bitlinear_forward_rmsnorm
 * does (the listing's per-BitLinear nn.RMSNorm).
 * Decode batches (M <= 6, and M K <= 196608, 2 M K with gate/up gains):
 * one GEMV launch streams the gate and up weights together (a CTA holds the
 * same rows of both), applies the quantised tokens to both and writes h from
 * its epilogue. Larger batches: gate and up as one grouped quantisation +
 * tensor-core launch pair (bitlinear_forward_grouped_ws, each with its own
 * gains), then a small kernel computes h from their bf16 outputs (the same
 * values). Then the down projection runs on h as bitlinear_forward_rmsnorm
 * (or bitlinear_forward without a down gain) does, GEMV or tensor cores by M.
 *   x_dev           [in]  [M][K] activations of type xdt
 *   M, K, F         [in]  tokens, d_model, d_ff; K and F positive multiples
 *                         of 128, at most 65536, else BITLINEAR_ERR_SHAPE
 *   gate_packed_dev, gate_gamma, up_packed_dev, up_gamma
 *                   [in]  F x K packed weights and their gammas
 *   down_packed_dev, down_gamma
 *                   [in]  K x F packed weights and gamma
 *   gate_gain_dev, up_gain_dev
 *                   [in]  [K] fp32 RMSNorm gains, both or neither (NULL:
 *                         no normalisation), 16-byte aligned
 *   down_gain_dev   [in]  [F] fp32 gains of the down projection, or NULL
 *   norm_eps        [in]  eps of the normalisations (finite, > 0) when any
 *                         gain is given; ignored otherwise
 *   h_dev           [out] [M][F] fp32, 16-byte aligned (the down input)
 *   y_dev           [out] [M][K] bf16
 *   workspace_dev, workspace_bytes
 *                   [in]  scratch of bitlinear_workspace_bytes_ffn(M, K, F)
 *                         bytes, 256-byte aligned (may be NULL when that
 *                         is 0)
 *   gate_y_dev_or_null, up_y_dev_or_null
 *                   [out, optional] [M][F] bf16 gate and up outputs
 * Errors as for bitlinear_forward, all reported before any launch. */
int bitlinear_ffn_forward(const void *x_dev, bitlinear_dtype xdt, int64_t M,
                          int64_t K, int64_t F, const void *gate_packed_dev,
                          float gate_gamma, const void *up_packed_dev,
                          float up_gamma, const void *down_packed_dev,
                          float down_gamma, const float *gate_gain_dev,
                          const float *up_gain_dev, const float *down_gain_dev,
                          float norm_eps, float *h_dev, void *y_dev,
                          void *workspace_dev, size_t workspace_bytes,
                          void *cuda_stream, void *gate_y_dev_or_null,
                          void *up_y_dev_or_null);

/* One problem of bitlinear_forward_grouped. */
typedef struct {
    const void *x_dev;       /* [M][K] activations (the group's xdt) */
    int64_t M, K, N;
    const void *packed_dev;  /* packed weights, bitlinear_packed_bytes(N, K) bytes */
    float gamma;             /* gamma from bitlinear_pack_weights */
    void *y_dev;             /* [M][N] bf16 output */
} bitlinear_problem;

/* Several independent BitLinear matmuls in one launch of the GEMV kernel,
 * for example the q/k/v or the gate/up projections of a decoder layer (which
 * may share x_dev), or any set of small-batch problems that do not depend on
 * each other's outputs. Each problem is computed exactly as bitlinear_forward
 * computes it on its own; grouping only shares one launch, and the CTAs of
 * every problem stream about the same number of weight bytes.
 *   problems [in] host array of count descriptors (1 <= count <= 8); every
 *                 problem needs the GEMV limits of bitlinear_forward_ex, and
 *                 the group's largest M * K must be within the limit of its
 *                 largest M (one launch holds both); M = 0 problems are
 *                 skipped
 *   xdt      [in] activation dtype of all problems
 * No workspace is needed. Outputs must not overlap each other or any input.
 * Argument errors are reported before any launch, as for bitlinear_forward. */
int bitlinear_forward_grouped(const bitlinear_problem *problems, int count,
                              bitlinear_dtype xdt, void *cuda_stream);

/* bitlinear_forward_grouped with base-3 packed weights
 * (bitlinear_pack_weights_b3) for every problem: one GEMV launch, each
 * problem computed exactly as bitlinear_forward_b3 computes it alone.
 *   problems [in] as for bitlinear_forward_grouped, packed_dev holding
 *                 bitlinear_packed_bytes_b3(N, K) bytes; M <= 16 and M * Kp
 *                 <= 196608 per problem (Kp = K rounded up to a multiple of
 *                 160), and the group's largest M * Kp within the limit of
 *                 its largest M
 *   xdt      [in] activation dtype of all problems
 * Errors as for bitlinear_forward_grouped, all reported before any launch. */
int bitlinear_forward_grouped_b3(const bitlinear_problem *problems, int count,
                                 bitlinear_dtype xdt, void *cuda_stream);

/* bitlinear_forward_grouped with the tokens taken from, and the outputs
 * returned to, host memory, all on cuda_stream. This is the one call a
 * decode step makes when its tokens arrive from the host and its outputs
 * leave for it.
 *   problems, count, xdt [in] as for bitlinear_forward_grouped; x_dev and
 *                  y_dev are the device staging buffers (caller-owned)
 *   x_host [in]  problem 0's M*K tokens (xdt elements, row-major), then
 *                problem 1's, and so on: sum of M*K elements
 *   y_host [out] problem 0's M*N bf16 outputs, then problem 1's, and so on
 * Tokens: when x_host is pinned memory mapped into the device's address
 * space (as cudaHostAlloc / cudaMallocHost memory is under unified
 * addressing), a small kernel reads it and writes every problem's x_dev;
 * otherwise cudaMemcpyAsync copies them (one copy for problems whose x_dev
 * buffers lie back to back). Outputs: when y_host is such memory and every
 * problem's part of it is 16-byte aligned, the GEMV writes the outputs
 * straight into y_host and y_dev is not written; otherwise the outputs go
 * to y_dev and cudaMemcpyAsync copies them back. The call returns once the
 * work is enqueued; y_host holds the results after the stream synchronises,
 * and x_host must keep this call's tokens until then. With pageable host
 * buffers CUDA makes the copies synchronous.
 * Errors: those of bitlinear_forward_grouped, reported before any copy or
 * launch; BITLINEAR_ERR_ARG for a NULL host buffer; BITLINEAR_ERR_CUDA when
 * a copy or the launch cannot be enqueued (earlier parts may be enqueued). */
int bitlinear_forward_grouped_host(const bitlinear_problem *problems, int count,
                                   bitlinear_dtype xdt, const void *x_host,
                                   void *y_host, void *cuda_stream);

/* Device workspace bytes bitlinear_forward_grouped_ws needs for these
 * problems: 0 when every non-empty problem takes the GEMV path on its own
 * (M <= 6 and M * K <= 196608; one GEMV launch),
 * else the sum of each problem's x~, beta and row-sum regions plus one
 * inter-CTA region (see bitlinear_workspace_bytes). SIZE_MAX for invalid
 * problems. */
size_t bitlinear_workspace_bytes_grouped(const bitlinear_problem *problems,
                                         int count);

/* Several independent BitLinear matmuls, at any batch size, in one pair of
 * launches. When every non-empty problem takes the GEMV path on its own
 * (M <= 6 and M * K <= 196608) this is
 * bitlinear_forward_grouped (one GEMV launch, the workspace is not used).
 * Otherwise all of them go to the tensor-core path: one quantisation launch
 * for every problem's tokens, then one weight-stationary GEMM launch over
 * all problems' tiles (stream-K across the problems), so the fixed cost of
 * the two launches is paid once for the group. Each problem's y is the same
 * as bitlinear_forward computes for it alone.
 *   problems, count, xdt [in] as for bitlinear_forward_grouped (no GEMV size
 *                        limit here)
 *   workspace_dev, workspace_bytes
 *               [in]  scratch of at least bitlinear_workspace_bytes_grouped
 *                     bytes, 256-byte aligned; not shared with a call that
 *                     may run at the same time
 * Errors as for bitlinear_forward; argument errors are reported before any
 * launch. */
int bitlinear_forward_grouped_ws(const bitlinear_problem *problems, int count,
                                 bitlinear_dtype xdt, void *workspace_dev,
                                 size_t workspace_bytes, void *cuda_stream);

/* bitlinear_forward_grouped_ws with every problem's tokens RMS-normalised
 * first (bitlinear_forward_rmsnorm's normalisation), each problem with its
 * own gains: for example the seven projections of a decoder layer, each
 * BitLinear with its own nn.RMSNorm as in the page's listing.
 *   problems, count, xdt, workspace_dev, workspace_bytes, cuda_stream
 *                  as for bitlinear_forward_grouped_ws (the same workspace
 *                  size, bitlinear_workspace_bytes_grouped)
 *   norm_gains_dev [in] host array of count device pointers, the [K] fp32
 *                  gains of each problem (16-byte aligned; NULL only for a
 *                  problem with M = 0)
 *   norm_eps       [in] finite and > 0
 * One GEMV launch when every problem takes the GEMV path on its own, else
 * one grouped quantisation launch (which normalises) and one GEMM launch.
 * Argument errors are reported before any launch. */
int bitlinear_forward_grouped_rmsnorm(const bitlinear_problem *problems,
                                      const float *const *norm_gains_dev,
                                      int count, float norm_eps,
                                      bitlinear_dtype xdt, void *workspace_dev,
                                      size_t workspace_bytes, void *cuda_stream);

/* Workspace bytes for an explicit path (see bitlinear_forward_ex); SIZE_MAX
 * for invalid shapes, including those BITLINEAR_PATH_GEMV cannot take. */
size_t bitlinear_workspace_bytes_path(int64_t M, int64_t N, int64_t K,
                                      int path);

/* Bytes of the device array that bitlinear_forward_noalloc uses as scratch. */
#define BITLINEAR_STATIC_SCRATCH_BYTES (16u << 20)

/* bitlinear_forward on the tensor-core path, for callers that cannot
 * allocate device memory themselves: for instance a plugin whose host hands
 * it only the input and output pointers and offers no allocator or workspace,
 * or a serving loop that forbids allocation once it has started. Nothing is
 * allocated by anyone. The scratch the path needs (x~, beta and the per-token
 * sums of x~; the GEMM then gives every CTA whole tiles, so it needs no
 * partial-sum region) lives in one file-scope device array of
 * BITLINEAR_STATIC_SCRATCH_BYTES (16 MiB) inside the library; every GPU that
 * loads the library holds that array until the process exits.
 * The method itself has no such call; it exists only for such callers.
 *   x_dev, packed_dev, gamma, y_dev, cuda_stream: as for bitlinear_forward.
 * Limits: M * K rounded up to 256 bytes, plus 2 * (4 * M rounded up to 256)
 * bytes, must fit in BITLINEAR_STATIC_SCRATCH_BYTES; larger problems return
 * BITLINEAR_ERR_SCRATCH_LIMIT before any device work (the largest M is
 * 6533 for K = 2560, 2424 for K = 6912, 2046 for K = 8192, 584 for K = 28672).
 * Set-up: the first call on a device (with that device current) looks up the
 * array's device address once; make that first call before any stream
 * capture.
 * Sharing: every call on a device uses the same array and it keeps the last
 * call's contents. Nothing in it needs to start at zero (each call writes
 * every scratch byte it reads before reading it), but calls whose work
 * overlaps on the GPU (different streams, or different host threads) race on
 * the array: serialise them, e.g. on one stream. */
int bitlinear_forward_noalloc(const void *x_dev, bitlinear_dtype xdt, int64_t M,
                              int64_t K, const void *packed_dev, float gamma,
                              int64_t N, void *y_dev, void *cuda_stream);

/* ------------------------------------------------------------- diagnostics */

/* Device-side fault word. Every bounded wait in the tensor-core GEMM gives
 * up after a time limit, records a nonzero code here and lets the kernel
 * return instead of hanging. This call synchronises cuda_stream, stores the
 * word in *fault_out (0 = none) and clears it. Returns BITLINEAR_ERR_TIMEOUT
 * when the word was set, BITLINEAR_ERR_CUDA when the synchronisation failed,
 * BITLINEAR_OK otherwise. */
int bitlinear_get_fault(int *fault_out, void *cuda_stream);

/* Human-readable name of a bitlinear_status. Never NULL. */
const char *bitlinear_status_string(int status);

/* ------------------------------------------------- failure-detection aids */

/* A forward with one wait made to run out on purpose, for the
 * failure-detection test. path selects the kernel (BITLINEAR_PATH_GEMV or
 * BITLINEAR_PATH_TC; anything else is BITLINEAR_ERR_ARG):
 *   - GEMV: the weight producer leaves the first stage unloaded, so the
 *     compute warps' first wait gives up after timeout_us microseconds;
 *   - TC: the MMA issuer waits on a barrier nobody arrives at, for
 *     timeout_us microseconds.
 * The kernel then records a fault (read by bitlinear_get_fault), every role
 * returns, and y is not written. Other inputs as for bitlinear_forward_ex
 * with that path; timeout_us in [1, 10^7]. */
int bitlinear_forward_inject_timeout(const void *x_dev, bitlinear_dtype xdt,
                                     int64_t M, int64_t K,
                                     const void *packed_dev, float gamma,
                                     int64_t N, void *y_dev,
                                     void *workspace_dev,
                                     size_t workspace_bytes,
                                     void *cuda_stream, int path,
                                     int timeout_us);

#ifdef __cplusplus
}
#endif

#endif /* BITLINEAR_H */
