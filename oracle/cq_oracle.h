/*
 * cq_oracle.h -- plain, slow, fp64 CPU oracle for Cactus-Quants (CQ) group-wise
 * Hadamard/codebook weight quantization.
 *
 * TEST INFRASTRUCTURE ONLY.  This oracle exists to check the CUDA library.  Only the
 * test suite, the smoke check and the CPU-baseline leg of the benchmark may load it;
 * the product path never calls it and shares no code, header or table with it.
 *
 * What it follows ("Cactus Quants CQ2-bit Quantization" = page 1, "How CQ2-bit
 * Quantization Contributes to Needle 2's Small Footprint" = page 2, "Performance
 * Differences Between 2-Bit and 4-Bit Quantization in Needle" = page 3, "How
 * Quantization Codebooks Are Trained in Cactus Quants" = page 4):
 *   - groups of 128 along the last axis, zero padded   (page 1, "Group-wise Weight
 *     Partitioning" and "The CQ2-bit Implementation Pipeline" steps 1 and 6)
 *   - orthonormal Walsh-Hadamard rotation               (page 1 "Hadamard Rotation";
 *     page 2 "Hadamard Rotation")
 *   - normalisation by the group's L2 norm, stored fp16 (page 2 "Per-Group Storage
 *     Breakdown")
 *   - nearest codebook entry                            (page 1 pipeline step 4)
 *   - Lloyd-Max Gaussian codebook / ternary constant    (page 4 "The Lloyd-Max
 *     Algorithm Implementation", "Ternary Special Case Handling", "Production Codebook
 *     Generation and Caching")
 *   - index bit-packing, norms stored separately        (page 2 "Binary Serialization")
 *   - dequantise = codeword x norm, inverse rotate, unpad (page 1 pipeline steps 5-6)
 *   - the fused GEMV is checked as explicit dequantise-then-matmul.
 *
 * Parity status of every function is listed beside it; each one is pinned by the
 * "not gpu" tests against closed forms, library routines or values the pages print.
 */
#ifndef CQ_ORACLE_H
#define CQ_ORACLE_H

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

/* Element types the oracle reads and writes (values match the library's enum). */
#define CQO_F32 0
#define CQO_BF16 1
#define CQO_F64 2

/* bits = 0 selects the ternary codebook, stored in 2-bit fields. */
#define CQO_TERNARY 0

/* Dense orthonormal Sylvester Walsh-Hadamard matrix, H[i*g+k] = (-1)^popcount(i&k)/sqrt(g).
 * g must be a power of two.  Returns 0, or -1 on a bad g.  (pinned: H_int H_int^T = g I,
 * Sylvester recursion, scipy.linalg.hadamard) */
int cqo_hadamard(int g, double* H);

/* MT19937 as NumPy's legacy RandomState(seed): raw 32-bit outputs, 53-bit doubles and the
 * polar-method normal deviates that randn() returns.  (pinned bit-exactly to NumPy) */
void cqo_mt_uint32(uint32_t seed, size_t n, uint32_t* out);
void cqo_randn(uint32_t seed, size_t n, double* out);

/* Lloyd-Max (1-D k-means) on sorted RandomState(seed).randn(samples): quantile
 * initialisation, `iters` rounds of midpoint boundaries / left-searchsorted assignment /
 * cell means, result sorted ascending (page 4).  levels >= 2.  (pinned: closed-form
 * Gaussian Lloyd-Max levels, the ternary constant, brute-force k-means) */
int cqo_lloyd_max(int levels, int samples, int iters, uint32_t seed, double* out);

/* Same iteration on caller data (already sorted ascending), for brute-force pins. */
int cqo_lloyd_on_sorted(const double* x, int n, int levels, int iters, double* out);

/* Codebook for `bits` in {0 (ternary), 2, 3, 4}: Lloyd-Max(2^bits levels, 400000 samples,
 * 200 iterations, seed) or the ternary constant, divided by sqrt(group_size) in fp64 and
 * rounded to fp32.  Writes n_levels floats; returns the level count or -1. */
int cqo_codebook(int bits, int group_size, uint32_t seed, float* out);

/* Number of levels for `bits` (3 for ternary), bits per stored index (2 for ternary). */
int cqo_levels(int bits);
int cqo_field_bits(int bits);

/* Byte counts: index stream rows*G*(g*field_bits/8), fp16 norms 2*rows*G, G = ceil(cols/g). */
size_t cqo_packed_bytes(int64_t rows, int64_t cols, int bits, int group_size);
size_t cqo_norm_bytes(int64_t rows, int64_t cols, int group_size);

/* fp64 -> fp16 / bf16 with round-to-nearest-even, overflow to inf.  (pinned: NumPy's
 * float16 conversion; hand-checked bf16 halfway cases) */
uint16_t cqo_f64_to_f16(double x);
double cqo_f16_to_f64(uint16_t h);
uint16_t cqo_f64_to_bf16(double x);

/* Quantise a row-major [rows, cols] matrix (dtype CQO_F32 or CQO_BF16) in groups of
 * group_size along cols.  For each group: zero pad, r = H v (dense fp64 product),
 * n = ||r||_2, u = r/n (0 when n == 0), idx_i = argmin_k |u_i - c_k| with ties to the
 * lower k, norm = fp16_rne(n), pack idx LSB-first.  Output: packed[rows*G*(g*b/8)] and
 * norms[rows*G] (fp16 bits).  Optionally also returns the fp64 normalised components
 * u_out[rows*G*g] (NULL to skip) for boundary-band checks.  nthreads <= 0: all cores. */
int cqo_quantize(const void* w, int dtype, int64_t rows, int64_t cols, int bits, int group_size,
                 const float* codebook, uint8_t* packed, uint16_t* norms, double* u_out,
                 int nthreads);

/* Dequantise: w_hat = H (fp64(norm16) * c[idx]) per group, unpadded, into fp64
 * out[rows*cols].  Codes >= n_levels decode as the top level. */
int cqo_dequantize(const uint8_t* packed, const uint16_t* norms, int64_t rows, int64_t cols,
                   int bits, int group_size, const float* codebook, double* out, int nthreads);

/* y[b, r] = sum_c W_hat[r, c] * x[b, c] with W_hat from cqo_dequantize (explicit, fp64)
 * and x of dtype CQO_F32 or CQO_BF16, shape [batch, cols].  y is fp64 [batch, rows]. */
int cqo_dequant_gemv(const uint8_t* packed, const uint16_t* norms, int64_t rows, int64_t cols,
                     int bits, int group_size, const float* codebook, const void* x, int x_dtype,
                     int batch, double* y, int nthreads);

/* Unpack the index of element i of group block `blk` (field_bits wide, LSB first). */
int cqo_unpack_index(const uint8_t* blk, int field_bits, int i);

/* Relative MSE sum((w - w_hat)^2) / sum(w^2) over the real elements. */
double cqo_rel_mse(const void* w, int dtype, const double* w_hat, int64_t n);

/* Threads the oracle uses when nthreads <= 0. */
int cqo_default_threads(void);

#ifdef __cplusplus
}
#endif
#endif
