/*
 * cq.h -- C ABI of libcq: Cactus-Quants (CQ) group-wise Hadamard/codebook weight
 * quantisation on NVIDIA B200 (sm_100a).
 *
 * The method (pages "Cactus Quants CQ2-bit Quantization" and "How CQ2-bit Quantization
 * Contributes to Needle 2's Small Footprint"): split each row of a weight matrix into
 * groups of 128 consecutive elements (zero padding the last one), rotate every group by
 * the orthonormal Sylvester Walsh-Hadamard matrix H (H[i][k] = (-1)^popcount(i&k)/sqrt(128)),
 * store the group's L2 norm as fp16, map each normalised component to the nearest entry of
 * a Gaussian Lloyd-Max codebook scaled by 1/sqrt(128), and bit-pack the indices.
 * Dequantisation multiplies codeword by norm, rotates back (H is its own inverse) and
 * drops the padding.
 *
 * Conventions shared by every call
 * --------------------------------
 *   Shapes    W is row-major [rows, cols]; groups run along cols; G = ceil(cols / 128)
 *             groups per row.  Only group_size == 128 is implemented (CQ_ERR_UNSUPPORTED
 *             otherwise), the pages' default.
 *   bits      CQ_BITS_TERNARY (0, the "1.58-bit" three-level codebook, stored in 2-bit
 *             fields), 2, 3 or 4.  L = 3, 4, 8 or 16 levels.
 *   Packed    Group (r, j) owns the 16*b bytes at offset (r*G + j)*16*b, b = field bits
 *   layout    (2 for ternary).  Index i of the group sits at bits [b*i, b*i + b) of that
 *             little-endian bitstream (LSB first).  Norms are a separate fp16 [rows, G]
 *             array (IEEE binary16 bit patterns, round to nearest even).  (Page "How
 *             CQ2-bit Quantization Contributes to Needle 2's Small Footprint", "Per-Group
 *             Storage Breakdown" and "Binary Serialization".)
 *   Codebook  `codebook` is a DEVICE pointer to L fp32 values sorted ascending and already
 *             scaled by 1/sqrt(128), or NULL for the built-in default (Lloyd-Max seed 0,
 *             or the ternary constant).  The first call with NULL for a given bit width
 *             on a device computes that default on the host and copies it to the device
 *             synchronously; make that first call before any stream capture.
 *   Memory    The caller allocates and owns every buffer.  The library allocates nothing
 *             per call.  All device pointers must be 16-byte aligned.
 *   Streams   `stream` is a cudaStream_t (NULL = legacy default stream).  Compute calls
 *             are asynchronous: they enqueue kernels and return without synchronising.
 *   Empty     rows == 0 or cols == 0 is valid: quantise / dequantise do nothing (their
 *             pointers may then be NULL) and the GEMV writes y = 0 (rows * batch zeros).
 *   Errors    Arguments are validated on the host before anything is launched; a bad
 *             argument returns an error and launches nothing.  A failed launch returns
 *             CQ_ERR_CUDA.  Kernels never trap: codes beyond the last level (ternary
 *             code 3) decode as the last level, and every wait inside a kernel is bounded
 *             (cq_device_status reports one that gave up).
 *   Threads   Calls may come from several host threads; each call uses the device that
 *             is current on the calling thread.
 */
#ifndef CQ_H
#define CQ_H

#include <stddef.h>

#ifdef __cplusplus
extern "C" {
#endif

typedef enum {
    CQ_OK = 0,
    CQ_ERR_INVALID_ARG = 1, /* null pointer, non-positive size, bad bits / dtype / batch  */
    CQ_ERR_UNSUPPORTED = 2, /* valid per the method but not implemented (group_size != 128) */
    CQ_ERR_CUDA = 3,        /* a CUDA runtime call or kernel launch failed                  */
    CQ_ERR_ALIGNMENT = 4,   /* a device pointer is not 16-byte aligned                      */
    CQ_ERR_WORKSPACE = 5    /* workspace missing or smaller than the size the library asks  */
} cq_status;

typedef enum {
    CQ_F32 = 0,  /* IEEE binary32 */
    CQ_BF16 = 1  /* bfloat16 (top half of a binary32), round to nearest even on output */
} cq_dtype;

#define CQ_BITS_TERNARY 0
#define CQ_GROUP_SIZE 128

/* Human-readable name of a status code.  Never NULL; static storage. */
const char* cq_status_string(int status);

/* Library version as 10000*major + 100*minor + patch. */
int cq_version(void);

/*
 * cq_device_status -- watchdog word of the current device.
 *
 * The tensor-core kernels coordinate their warps through shared-memory barriers; every wait
 * on one gives up after a few seconds instead of spinning forever, sets bit 0 of this word,
 * and the kernel returns early (its outputs are then incomplete).  This call copies the
 * word to *status_out (0 = no wait ever gave up) and clears it when `reset` is nonzero.
 * It synchronises with the device (a blocking copy), so it is a diagnostic, not for hot
 * paths.  Returns CQ_OK, CQ_ERR_INVALID_ARG (status_out NULL) or CQ_ERR_CUDA.
 */
int cq_device_status(int reset, unsigned* status_out);

/*
 * cq_codebook -- the default codebook for `bits` (host routine, setup only).
 *
 * Page "How Quantization Codebooks Are Trained in Cactus Quants": Lloyd-Max (1-D k-means)
 * on sorted NumPy-legacy RandomState(seed).randn(400000) samples, quantile initialisation
 * c_k = x[int((k + 0.5)/L * N)], 200 rounds of midpoint boundaries, left-searchsorted
 * assignment and cell means, sorted; ternary returns the hard-coded [-1.2240064, 0,
 * 1.2240064] ("Ternary Special Case Handling").  The levels are divided by
 * sqrt(group_size) in fp64 and rounded to fp32 ("Production Codebook Generation and
 * Caching").  Results are memoised per (bits, group_size, seed).
 *
 *   bits        CQ_BITS_TERNARY, 2, 3 or 4
 *   group_size  power of two in [8, 4096]
 *   seed        RandomState seed (the pages' default is 0); ignored for ternary
 *   out_host    HOST buffer of at least 16 floats; receives L values, ascending
 *   n_levels    HOST int* receiving L (may be NULL)
 * Returns CQ_OK or CQ_ERR_INVALID_ARG.  Touches no GPU.
 */
int cq_codebook(int bits, int group_size, unsigned long long seed, float* out_host,
                int* n_levels);

/*
 * Byte counts of the two stored arrays (page "How CQ2-bit Quantization Contributes to
 * Needle 2's Small Footprint", "Per-Group Storage Breakdown": b bits per weight for the
 * index plus one 16-bit norm per group, nothing else).
 *   cq_packed_bytes = rows * G * group_size * b / 8      (index stream only)
 *   cq_norm_bytes   = 2 * rows * G
 * Return 0 for invalid arguments (and for empty shapes).
 */
size_t cq_packed_bytes(long long rows, long long cols, int bits, int group_size);
size_t cq_norm_bytes(long long rows, long long cols, int group_size);

/*
 * cq_quantize -- quantise W to packed indices and fp16 norms.
 *
 * Page "Cactus Quants CQ2-bit Quantization", "The CQ2-bit Implementation Pipeline"
 * steps 1-4 (pad and reshape, rotate, normalise, nearest-codeword lookup), with the
 * stored form of page "How CQ2-bit Quantization Contributes to Needle 2's Small
 * Footprint", "Binary Serialization".  Per group: v zero padded, r = H v, n = ||r||_2,
 * u = r / n (u = 0 when n = 0), idx_i = the nearest codeword with ties to the lower
 * index (decided against fp32 midpoints), norm = fp16(n).
 *
 *   w           DEVICE [rows, cols] of w_dtype, row-major, contiguous
 *   w_dtype     CQ_F32 or CQ_BF16
 *   rows, cols  >= 0
 *   bits        CQ_BITS_TERNARY, 2, 3 or 4
 *   group_size  must be 128
 *   codebook    DEVICE L fp32 ascending, or NULL for the default
 *   packed_out  DEVICE cq_packed_bytes(rows, cols, bits, 128) bytes, written fully
 *   norms_out   DEVICE cq_norm_bytes(rows, cols, 128) bytes (fp16 bit patterns)
 *   stream      cudaStream_t or NULL
 * Returns CQ_OK after enqueueing, or an error with nothing launched.
 */
int cq_quantize(const void* w, int w_dtype, long long rows, long long cols, int bits,
                int group_size, const float* codebook, unsigned char* packed_out,
                unsigned short* norms_out, void* stream);

/*
 * cq_quantize_batch -- cq_quantize over a list of tensors in as few launches as possible.
 *
 * Same arithmetic and results as calling cq_quantize on every job in order on `stream`
 * (same w_dtype, bits, group size and codebook for all).  Quantising a whole model is this
 * call: the tensors are processed together, so no launch waits for the previous tensor's
 * last tile.  Because the jobs run concurrently, no job's outputs may overlap another job's
 * input or outputs.
 *
 *   jobs        HOST array of `count` descriptors, read during the call only; each job
 *               follows cq_quantize's rules for w, rows, cols, packed_out and norms_out
 *   count       >= 0 (0: nothing to do)
 * Every job is validated before anything is launched; the first failing job's status is
 * returned.  Returns CQ_OK after enqueueing.
 */
typedef struct cq_quantize_job {
    const void* w;
    long long rows;
    long long cols;
    unsigned char* packed_out;
    unsigned short* norms_out;
} cq_quantize_job;

int cq_quantize_batch(const cq_quantize_job* jobs, int count, int w_dtype, int bits,
                      int group_size, const float* codebook, void* stream);

/*
 * cq_dequantize -- reconstruct W_hat from packed indices and fp16 norms.
 *
 * Page "Cactus Quants CQ2-bit Quantization", "The CQ2-bit Implementation Pipeline"
 * steps 5-6 (inverse rotate, unpad) and page "How Needle 2 Compresses to a Single
 * Binary", "Stage 3" (the runtime reconstructs the 2-bit tensors on the fly):
 * w_hat = H (fp32(norm16) * c[idx]) per group, padding columns dropped.
 *
 *   packed, norms  DEVICE, as written by cq_quantize
 *   rows, cols     >= 0, the shape of W
 *   bits, group_size, codebook   as for cq_quantize
 *   out            DEVICE [rows, cols] of out_dtype, row-major, contiguous
 *   out_dtype      CQ_F32 or CQ_BF16 (bf16 rounds the fp32 result to nearest even)
 */
int cq_dequantize(const unsigned char* packed, const unsigned short* norms, long long rows,
                  long long cols, int bits, int group_size, const float* codebook, void* out,
                  int out_dtype, void* stream);

/*
 * cq_dequantize_batch -- cq_dequantize over a list of tensors in as few launches as
 * possible.  Same results as calling cq_dequantize on every job in order on `stream` (same
 * bits, group size, codebook and out_dtype for all).  The jobs run concurrently, so no job's
 * output may overlap another job's inputs or output.
 *
 *   jobs        HOST array of `count` descriptors, read during the call only; each job
 *               follows cq_dequantize's rules for packed, norms, rows, cols and out
 *   count       >= 0 (0: nothing to do)
 * Every job is validated before anything is launched; the first failing job's status is
 * returned.  Returns CQ_OK after enqueueing.
 */
typedef struct cq_dequantize_job {
    const unsigned char* packed;
    const unsigned short* norms;
    long long rows;
    long long cols;
    void* out;
} cq_dequantize_job;

int cq_dequantize_batch(const cq_dequantize_job* jobs, int count, int bits, int group_size,
                        const float* codebook, int out_dtype, void* stream);

/*
 * cq_fake_quantize -- W_hat = dequantize(quantize(W)) in one call: the tensor that the
 * pages' cq_quantize returns.
 *
 * Page "Cactus Quants CQ2-bit Quantization", "The CQ2-bit Implementation Pipeline" steps
 * 1-6 (pad, rotate, normalise, nearest codeword, inverse rotate, unpad), whose output is the
 * de-quantised tensor; page "How Quantization Codebooks Are Trained in Cactus Quants",
 * "Practical Usage Example" (cq_quantize applied with a caller codebook).  The scale
 * used for the inverse rotation is the stored fp16 norm, so W_hat is bit for bit what
 * cq_dequantize reconstructs from the stored form that cq_quantize writes.
 *
 *   w, w_dtype, rows, cols, bits, group_size, codebook   as for cq_quantize
 *   packed_out, norms_out   DEVICE buffers as for cq_quantize; they receive the stored form
 *                           (the intermediate; the caller may discard it)
 *   out, out_dtype          as for cq_dequantize.  out may be w itself (in-place fake
 *                           quantisation, when the dtypes match): every read of w completes
 *                           before the first write of out.  It must not overlap packed_out
 *                           or norms_out.
 * Two launches on `stream` (quantise, then dequantise).  Every argument is validated before
 * anything is launched.  Returns CQ_OK after enqueueing, or an error with nothing launched.
 */
int cq_fake_quantize(const void* w, int w_dtype, long long rows, long long cols, int bits,
                     int group_size, const float* codebook, unsigned char* packed_out,
                     unsigned short* norms_out, void* out, int out_dtype, void* stream);

/*
 * cq_fake_quantize_batch -- cq_fake_quantize over a list of tensors: one cq_quantize_batch
 * over all jobs, then one cq_dequantize_batch.  Every w is read before any out is written,
 * so outputs may alias any job's w; otherwise the rules of the two batched calls apply (no
 * job's packed_out / norms_out may overlap another job's buffers or any out).
 *
 *   jobs        HOST array of `count` descriptors, read during the call only
 *   count       >= 0 (0: nothing to do)
 * Every job is validated before anything is launched; the first failing job's status is
 * returned.  Returns CQ_OK after enqueueing.
 */
typedef struct cq_fake_quantize_job {
    const void* w;
    long long rows;
    long long cols;
    unsigned char* packed_out;
    unsigned short* norms_out;
    void* out;
} cq_fake_quantize_job;

int cq_fake_quantize_batch(const cq_fake_quantize_job* jobs, int count, int w_dtype, int bits,
                           int group_size, const float* codebook, int out_dtype, void* stream);

/*
 * cq_dequant_gemv -- y = W_hat x without materialising W_hat.
 *
 * Because H is symmetric and orthonormal (page "How CQ2-bit Quantization Contributes to
 * Needle 2's Small Footprint", "Hadamard Rotation"; page "Cactus Quants CQ2-bit
 * Quantization", "Hadamard Rotation"), each activation group is rotated once,
 * x~_j = H x_j, and y[b, r] = sum_j fp32(norm16_rj) * <c[idx_rj], x~_bj>, accumulated in
 * fp32.  The memory-bandwidth motive is page "Performance Differences Between 2-Bit and
 * 4-Bit Quantization in Needle", "Model Size and Memory Bandwidth".
 *
 * Arithmetic: the products run on the tensor cores.  Each rotated activation group is
 * scaled by its own power of two (largest magnitude in [2^13, 2^14)) and the codewords by
 * one power of two per call.  2-bit and ternary codes: both are rounded to 16-bit integers
 * and multiplied exactly as two int8 planes each (int32 accumulation per group), the group's
 * four cross products being combined in fp32.  3/4-bit codes: both are rounded to fp16 and
 * multiplied with fp32 accumulation.  Any finite input is in range; the relative error of y
 * is about 3e-4 (bound 1e-3 per output vector).  Summation order is fixed: repeated calls
 * give identical bits.
 *
 *   packed, norms  DEVICE, W quantised as [rows, cols] (rows = outputs, cols = inputs)
 *   rows, cols     >= 0
 *   bits           CQ_BITS_TERNARY, 2, 3 or 4
 *   group_size     must be 128
 *   codebook       DEVICE L fp32 ascending, or NULL for the default
 *   x              DEVICE bf16 [batch, cols], row-major
 *   batch          1..64.  The tensor cores take 8 activation rows at a time: a batch above 8
 *                  runs as ceil(batch / 8) blocks of at most 8 rows in the same launches,
 *                  each block streaming the packed weights again (from L2 while they stay
 *                  resident), so HBM traffic for the weights grows with ceil(batch / 8).
 *   y              DEVICE fp32 [batch, rows], row-major, overwritten
 *   workspace      DEVICE scratch of at least cq_gemv_workspace_bytes(cols, batch) bytes
 *                  (2080 bytes per 128 columns plus 48, rounded up to 256, per block of 8
 *                  activation rows), 16-byte aligned; its contents on entry are ignored and
 *                  on return are unspecified.  Calls that overlap in time must not share a
 *                  workspace.
 */
int cq_dequant_gemv(const unsigned char* packed, const unsigned short* norms, long long rows,
                    long long cols, int bits, int group_size, const float* codebook,
                    const void* x, int batch, float* y, void* workspace,
                    size_t workspace_bytes, void* stream);

/*
 * cq_dequant_gemv_batch -- several independent cq_dequant_gemv products in one rotation
 * launch and one GEMV launch.  Same results as calling cq_dequant_gemv on every job in order
 * on `stream` (same bits, group size and codebook for all): the products run concurrently,
 * so no job's y or workspace may overlap anything another job reads or writes.
 *
 *   jobs        HOST array of `count` descriptors, read during the call only; each job
 *               follows cq_dequant_gemv's rules for its fields (its own workspace of at least
 *               cq_gemv_workspace_bytes(cols, batch) bytes)
 *   count       >= 0 (0: nothing to do)
 * Every job is validated before anything is launched; the first failing job's status is
 * returned.  Returns CQ_OK after enqueueing.
 */
typedef struct cq_gemv_job {
    const unsigned char* packed;
    const unsigned short* norms;
    long long rows;
    long long cols;
    const void* x;
    int batch;
    float* y;
    void* workspace;
    size_t workspace_bytes;
} cq_gemv_job;

int cq_dequant_gemv_batch(const cq_gemv_job* jobs, int count, int bits, int group_size,
                          const float* codebook, void* stream);

/* Workspace bytes cq_dequant_gemv needs for this cols and batch (0 if invalid or cols == 0). */
size_t cq_gemv_workspace_bytes(long long cols, int batch);

/*
 * cq_dequant_gemv_static -- cq_dequant_gemv without a workspace argument.
 *
 * No counterpart on the pages: this is a convenience of this library.  Some callers cannot
 * allocate device memory at the point where they need the product: code running while a
 * stream is being captured into a CUDA graph (cudaMalloc is not allowed then), plug-ins
 * that live inside a host framework and may not bypass its allocator, and C callers with
 * no device allocator of their own.  This entry point takes its scratch from a fixed array
 * in the library's own device memory (static, 532,736 bytes, held by every GPU that loads
 * the library until the process exits) and calls no cudaMalloc, cudaFree or allocating
 * routine.  Same arguments, semantics and results as cq_dequant_gemv, minus the workspace.
 *
 *   cols       at most 32768; larger returns CQ_ERR_WORKSPACE and launches nothing
 *   batch      1..64; the array holds one block of 8 activation rows, so a batch above 8
 *              runs as consecutive launch pairs on `stream`, one per block
 *   set-up     the first call on each device looks up the array's device address (a
 *              synchronous runtime call); make that first call before any stream capture
 *   sharing    every call on a device uses the same array, which keeps the last call's
 *              contents (nothing needs clearing: each call rewrites all it reads); calls
 *              whose executions overlap on the GPU, e.g. on two unordered streams, race.
 */
int cq_dequant_gemv_static(const unsigned char* packed, const unsigned short* norms,
                           long long rows, long long cols, int bits, int group_size,
                           const float* codebook, const void* x, int batch, float* y,
                           void* stream);

#ifdef __cplusplus
}
#endif
#endif /* CQ_H */
