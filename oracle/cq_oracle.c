/*
 * cq_oracle.c -- plain fp64 CPU oracle for CQ quantisation.  TEST INFRASTRUCTURE ONLY:
 * the product library never links or calls this file; only the tests, the smoke check
 * and the benchmark's CPU-baseline leg do.
 *
 * Everything here is written to be checked by eye against the method's description:
 * the rotation is an explicit dense 128x128 matrix product, the nearest search is brute
 * force over every codeword, the GEMV dequantises the whole matrix first.  No blocking,
 * no fusion, no fast transform.  Threads only split independent groups / rows.
 *
 * Parity: every function is pinned by the CPU tests (see the header for the pins).
 */
#define _GNU_SOURCE
#include "cq_oracle.h"

#include <math.h>
#include <pthread.h>
#include <stdlib.h>
#include <string.h>
#include <unistd.h>

/* ------------------------------------------------------------------------------------ */
/* small helpers                                                                         */
/* ------------------------------------------------------------------------------------ */

static int is_pow2(int g) { return g > 0 && (g & (g - 1)) == 0; }

static int popcount_u32(unsigned v) {
    int c = 0;
    while (v) { c += (int)(v & 1u); v >>= 1; }
    return c;
}

int cqo_default_threads(void) {
    long n = sysconf(_SC_NPROCESSORS_ONLN);
    return n > 0 ? (int)n : 1;
}

int cqo_levels(int bits) {
    if (bits == CQO_TERNARY) return 3;
    if (bits >= 2 && bits <= 4) return 1 << bits;
    return -1;
}

int cqo_field_bits(int bits) {
    if (bits == CQO_TERNARY) return 2; /* "1.58-bit" ternary codes live in 2-bit fields */
    if (bits >= 2 && bits <= 4) return bits;
    return -1;
}

static double load_elem(const void* w, int dtype, int64_t i) {
    if (dtype == CQO_F32) return (double)((const float*)w)[i];
    if (dtype == CQO_F64) return ((const double*)w)[i];
    /* bf16: the top 16 bits of an IEEE binary32 */
    uint32_t bits = ((uint32_t)((const uint16_t*)w)[i]) << 16;
    float f;
    memcpy(&f, &bits, 4);
    return (double)f;
}

/* ------------------------------------------------------------------------------------ */
/* Hadamard matrix (page 1 "Hadamard Rotation"; page 2 "Hadamard Rotation": an          */
/* orthonormal, parameter-free Walsh-Hadamard matrix).  Sylvester order.                 */
/* ------------------------------------------------------------------------------------ */

int cqo_hadamard(int g, double* H) {
    if (!is_pow2(g)) return -1;
    double s = 1.0 / sqrt((double)g);
    for (int i = 0; i < g; ++i)
        for (int k = 0; k < g; ++k)
            H[(size_t)i * g + k] = (popcount_u32((unsigned)(i & k)) & 1) ? -s : s;
    return 0;
}

/* ------------------------------------------------------------------------------------ */
/* MT19937 (Matsumoto & Nishimura, ACM TOMACS 1998) seeded the way NumPy's legacy        */
/* RandomState(int) seeds it, with NumPy's 53-bit double and polar-method gauss.         */
/* Page 4 "Gaussian Sampling and Initialization": samples come from                      */
/* RandomState(seed).randn(samples).                                                    */
/* ------------------------------------------------------------------------------------ */

typedef struct {
    uint32_t mt[624];
    int idx;
    int has_gauss;
    double gauss;
} mt_state;

static void mt_seed(mt_state* s, uint32_t seed) {
    s->mt[0] = seed;
    for (int i = 1; i < 624; ++i)
        s->mt[i] = 1812433253u * (s->mt[i - 1] ^ (s->mt[i - 1] >> 30)) + (uint32_t)i;
    s->idx = 624;
    s->has_gauss = 0;
    s->gauss = 0.0;
}

static void mt_twist(mt_state* s) {
    for (int i = 0; i < 624; ++i) {
        uint32_t y = (s->mt[i] & 0x80000000u) | (s->mt[(i + 1) % 624] & 0x7fffffffu);
        uint32_t v = s->mt[(i + 397) % 624] ^ (y >> 1);
        if (y & 1u) v ^= 0x9908b0dfu;
        s->mt[i] = v;
    }
    s->idx = 0;
}

static uint32_t mt_next(mt_state* s) {
    if (s->idx >= 624) mt_twist(s);
    uint32_t y = s->mt[s->idx++];
    y ^= y >> 11;
    y ^= (y << 7) & 0x9d2c5680u;
    y ^= (y << 15) & 0xefc60000u;
    y ^= y >> 18;
    return y;
}

/* 53-bit uniform in [0, 1): 27 high bits of one draw, 26 of the next. */
static double mt_double(mt_state* s) {
    uint32_t a = mt_next(s) >> 5, b = mt_next(s) >> 6;
    return ((double)a * 67108864.0 + (double)b) / 9007199254740992.0;
}

/* Marsaglia's polar method; each accepted pair returns f*x2 and caches f*x1. */
static double mt_gauss(mt_state* s) {
    if (s->has_gauss) {
        s->has_gauss = 0;
        return s->gauss;
    }
    double x1, x2, r2;
    do {
        x1 = 2.0 * mt_double(s) - 1.0;
        x2 = 2.0 * mt_double(s) - 1.0;
        r2 = x1 * x1 + x2 * x2;
    } while (r2 >= 1.0 || r2 == 0.0);
    double f = sqrt(-2.0 * log(r2) / r2);
    s->gauss = f * x1;
    s->has_gauss = 1;
    return f * x2;
}

void cqo_mt_uint32(uint32_t seed, size_t n, uint32_t* out) {
    mt_state s;
    mt_seed(&s, seed);
    for (size_t i = 0; i < n; ++i) out[i] = mt_next(&s);
}

void cqo_randn(uint32_t seed, size_t n, double* out) {
    mt_state* s = (mt_state*)malloc(sizeof(mt_state));
    mt_seed(s, seed);
    for (size_t i = 0; i < n; ++i) out[i] = mt_gauss(s);
    free(s);
}

/* ------------------------------------------------------------------------------------ */
/* Lloyd-Max (page 4 "Iterative Refinement of Quantization Levels").                     */
/* ------------------------------------------------------------------------------------ */

static int cmp_double(const void* a, const void* b) {
    double x = *(const double*)a, y = *(const double*)b;
    return (x > y) - (x < y);
}

/* Number of boundaries strictly below v: the position a left-sided searchsorted returns. */
static int searchsorted_left(const double* bnd, int nb, double v) {
    int i = 0;
    while (i < nb && bnd[i] < v) ++i;
    return i;
}

int cqo_lloyd_on_sorted(const double* x, int n, int levels, int iters, double* c) {
    if (levels < 2 || n < levels) return -1;
    /* quantile initialisation: c_k = x[int((k + 0.5) / L * N)] */
    for (int k = 0; k < levels; ++k) {
        double pos = ((double)k + 0.5) / (double)levels * (double)n;
        c[k] = x[(int64_t)pos];
    }
    double* bnd = (double*)malloc(sizeof(double) * (size_t)levels);
    double* sum = (double*)malloc(sizeof(double) * (size_t)levels);
    int64_t* cnt = (int64_t*)malloc(sizeof(int64_t) * (size_t)levels);
    for (int it = 0; it < iters; ++it) {
        /* decision boundaries: midpoints of consecutive levels */
        for (int k = 0; k + 1 < levels; ++k) bnd[k] = (c[k] + c[k + 1]) / 2.0;
        for (int k = 0; k < levels; ++k) { sum[k] = 0.0; cnt[k] = 0; }
        /* assignment of every sample, then cell means (an empty cell keeps its level) */
        for (int i = 0; i < n; ++i) {
            int k = searchsorted_left(bnd, levels - 1, x[i]);
            sum[k] += x[i];
            cnt[k] += 1;
        }
        for (int k = 0; k < levels; ++k)
            if (cnt[k] > 0) c[k] = sum[k] / (double)cnt[k];
    }
    qsort(c, (size_t)levels, sizeof(double), cmp_double);
    free(bnd);
    free(sum);
    free(cnt);
    return 0;
}

int cqo_lloyd_max(int levels, int samples, int iters, uint32_t seed, double* out) {
    if (levels < 2 || samples < levels) return -1;
    double* x = (double*)malloc(sizeof(double) * (size_t)samples);
    cqo_randn(seed, (size_t)samples, x);
    qsort(x, (size_t)samples, sizeof(double), cmp_double);
    int rc = cqo_lloyd_on_sorted(x, samples, levels, iters, out);
    free(x);
    return rc;
}

/* Page 4 "Ternary Special Case Handling" prints the constant; "Production Codebook
 * Generation and Caching" divides the Gaussian levels by sqrt(group_size). */
int cqo_codebook(int bits, int group_size, uint32_t seed, float* out) {
    int L = cqo_levels(bits);
    if (L < 0 || !is_pow2(group_size)) return -1;
    double lv[16];
    if (bits == CQO_TERNARY) {
        lv[0] = -1.2240064;
        lv[1] = 0.0;
        lv[2] = 1.2240064;
    } else if (cqo_lloyd_max(L, 400000, 200, seed, lv) != 0) {
        return -1;
    }
    double s = sqrt((double)group_size);
    for (int k = 0; k < L; ++k) out[k] = (float)(lv[k] / s);
    return L;
}

/* ------------------------------------------------------------------------------------ */
/* Sizes (page 2 "Per-Group Storage Breakdown": b bits per index plus one fp16 norm per  */
/* group of 128, nothing else).                                                          */
/* ------------------------------------------------------------------------------------ */

size_t cqo_packed_bytes(int64_t rows, int64_t cols, int bits, int group_size) {
    int fb = cqo_field_bits(bits);
    if (fb < 0 || group_size <= 0 || rows < 0 || cols < 0) return 0;
    int64_t G = (cols + group_size - 1) / group_size;
    return (size_t)(rows * G * ((int64_t)group_size * fb / 8));
}

size_t cqo_norm_bytes(int64_t rows, int64_t cols, int group_size) {
    if (group_size <= 0 || rows < 0 || cols < 0) return 0;
    int64_t G = (cols + group_size - 1) / group_size;
    return (size_t)(2 * rows * G);
}

/* ------------------------------------------------------------------------------------ */
/* Correctly rounded conversions from fp64 (round half to even).                          */
/* ------------------------------------------------------------------------------------ */

/* Round |x| to a multiple of 2^q with ties to even; exact because scaling by 2^-q is. */
static double round_to_quantum(double ax, int q) {
    double scaled = ldexp(ax, -q);
    double fl = floor(scaled);
    double rem = scaled - fl;
    if (rem > 0.5 || (rem == 0.5 && fmod(fl, 2.0) != 0.0)) fl += 1.0;
    return ldexp(fl, q);
}

uint16_t cqo_f64_to_f16(double x) {
    uint16_t sign = signbit(x) ? 0x8000u : 0u;
    if (isnan(x)) return 0x7e00u;
    double ax = fabs(x);
    if (isinf(ax)) return sign | 0x7c00u;
    if (ax == 0.0) return sign;
    int e;
    frexp(ax, &e);          /* ax = m * 2^e, m in [0.5, 1): unbiased exponent is e - 1 */
    int ue = e - 1;
    if (ue < -14) ue = -14; /* subnormals share the quantum 2^-24 */
    double r = round_to_quantum(ax, ue - 10);
    if (r >= 65520.0 || r > 65504.0) return sign | 0x7c00u;
    if (r < ldexp(1.0, -14)) return sign | (uint16_t)ldexp(r, 24); /* subnormal */
    frexp(r, &e);
    int be = e - 1 + 15;
    uint16_t mant = (uint16_t)(ldexp(r, -(e - 1)) * 1024.0 - 1024.0);
    return sign | (uint16_t)(be << 10) | mant;
}

double cqo_f16_to_f64(uint16_t h) {
    int s = (h >> 15) & 1, e = (h >> 10) & 31, m = h & 1023;
    double v;
    if (e == 0) v = ldexp((double)m, -24);
    else if (e == 31) v = m ? NAN : INFINITY;
    else v = ldexp(1.0 + m / 1024.0, e - 15);
    return s ? -v : v;
}

uint16_t cqo_f64_to_bf16(double x) {
    uint16_t sign = signbit(x) ? 0x8000u : 0u;
    if (isnan(x)) return 0x7fc0u;
    double ax = fabs(x);
    if (isinf(ax)) return sign | 0x7f80u;
    if (ax == 0.0) return sign;
    int e;
    frexp(ax, &e);
    int ue = e - 1;
    if (ue < -126) ue = -126;
    double r = round_to_quantum(ax, ue - 7);
    if (r >= ldexp(1.0, 128)) return sign | 0x7f80u;
    float f = (float)r; /* exact: r has at most 8 significant bits */
    uint32_t b;
    memcpy(&b, &f, 4);
    return sign | (uint16_t)((b >> 16) & 0x7fffu);
}

/* ------------------------------------------------------------------------------------ */
/* Bit packing (page 2 "Binary Serialization": consecutive indices packed into bytes,    */
/* fp16 norms kept apart).  Index i of a group occupies bits [b*i, b*i+b) of the group's */
/* little-endian bitstream.                                                               */
/* ------------------------------------------------------------------------------------ */

static void pack_index(uint8_t* blk, int fb, int i, int v) {
    for (int t = 0; t < fb; ++t) {
        int p = fb * i + t;
        if ((v >> t) & 1) blk[p / 8] |= (uint8_t)(1u << (p % 8));
    }
}

int cqo_unpack_index(const uint8_t* blk, int fb, int i) {
    int v = 0;
    for (int t = 0; t < fb; ++t) {
        int p = fb * i + t;
        v |= ((blk[p / 8] >> (p % 8)) & 1) << t;
    }
    return v;
}

/* ------------------------------------------------------------------------------------ */
/* Worker plumbing: split [0, n) into contiguous chunks, one per thread.                  */
/* ------------------------------------------------------------------------------------ */

typedef void (*range_fn)(void* ctx, int64_t begin, int64_t end);
typedef struct {
    range_fn fn;
    void* ctx;
    int64_t b, e;
} range_job;

static void* run_range(void* p) {
    range_job* j = (range_job*)p;
    j->fn(j->ctx, j->b, j->e);
    return NULL;
}

static void parallel_for(int64_t n, int nthreads, range_fn fn, void* ctx) {
    if (nthreads <= 0) nthreads = cqo_default_threads();
    if (nthreads > n) nthreads = (int)(n > 0 ? n : 1);
    if (nthreads <= 1) {
        fn(ctx, 0, n);
        return;
    }
    pthread_t* th = (pthread_t*)malloc(sizeof(pthread_t) * (size_t)nthreads);
    range_job* jobs = (range_job*)malloc(sizeof(range_job) * (size_t)nthreads);
    for (int t = 0; t < nthreads; ++t) {
        jobs[t].fn = fn;
        jobs[t].ctx = ctx;
        jobs[t].b = n * t / nthreads;
        jobs[t].e = n * (t + 1) / nthreads;
        pthread_create(&th[t], NULL, run_range, &jobs[t]);
    }
    for (int t = 0; t < nthreads; ++t) pthread_join(th[t], NULL);
    free(th);
    free(jobs);
}

/* ------------------------------------------------------------------------------------ */
/* Quantise (page 1 "The CQ2-bit Implementation Pipeline" steps 1-4; page 2 "Hadamard    */
/* Rotation" and "Per-Group Storage Breakdown").                                         */
/* ------------------------------------------------------------------------------------ */

typedef struct {
    const void* w;
    int dtype;
    int64_t rows, cols, G;
    int g, L, fb, blk_bytes;
    const double* H;
    const double* cb;
    uint8_t* packed;
    uint16_t* norms;
    double* u_out;
} quant_ctx;

static void quant_range(void* p, int64_t g0, int64_t g1) {
    quant_ctx* q = (quant_ctx*)p;
    int g = q->g;
    double* v = (double*)malloc(sizeof(double) * (size_t)g);
    double* r = (double*)malloc(sizeof(double) * (size_t)g);
    for (int64_t gid = g0; gid < g1; ++gid) {
        int64_t row = gid / q->G, j = gid % q->G;
        /* step 1: the group, zero padded past the last column */
        for (int i = 0; i < g; ++i) {
            int64_t col = j * g + i;
            v[i] = col < q->cols ? load_elem(q->w, q->dtype, row * q->cols + col) : 0.0;
        }
        /* step 2: rotate, r = H v (explicit dense product) */
        for (int i = 0; i < g; ++i) {
            double acc = 0.0;
            for (int k = 0; k < g; ++k) acc += q->H[(size_t)i * g + k] * v[k];
            r[i] = acc;
        }
        /* step 3: L2 norm of the rotated group; normalise */
        double ss = 0.0;
        for (int i = 0; i < g; ++i) ss += r[i] * r[i];
        double n = sqrt(ss);
        q->norms[gid] = cqo_f64_to_f16(n);
        uint8_t* blk = q->packed + gid * q->blk_bytes;
        memset(blk, 0, (size_t)q->blk_bytes);
        for (int i = 0; i < g; ++i) {
            double u = n > 0.0 ? r[i] / n : 0.0;
            if (q->u_out) q->u_out[gid * g + i] = u;
            /* step 4: nearest codeword, brute force, ties to the lower index */
            int best = 0;
            double bd = fabs(u - q->cb[0]);
            for (int k = 1; k < q->L; ++k) {
                double d = fabs(u - q->cb[k]);
                if (d < bd) { bd = d; best = k; }
            }
            pack_index(blk, q->fb, i, best);
        }
    }
    free(v);
    free(r);
}

int cqo_quantize(const void* w, int dtype, int64_t rows, int64_t cols, int bits, int group_size,
                 const float* codebook, uint8_t* packed, uint16_t* norms, double* u_out,
                 int nthreads) {
    int L = cqo_levels(bits), fb = cqo_field_bits(bits);
    if (L < 0 || !is_pow2(group_size) || group_size < 8 || rows < 0 || cols < 0) return -1;
    if (dtype != CQO_F32 && dtype != CQO_BF16 && dtype != CQO_F64) return -1;
    quant_ctx q;
    q.w = w;
    q.dtype = dtype;
    q.rows = rows;
    q.cols = cols;
    q.G = (cols + group_size - 1) / group_size;
    q.g = group_size;
    q.L = L;
    q.fb = fb;
    q.blk_bytes = group_size * fb / 8;
    double* H = (double*)malloc(sizeof(double) * (size_t)group_size * group_size);
    cqo_hadamard(group_size, H);
    double cb[16];
    for (int k = 0; k < L; ++k) cb[k] = (double)codebook[k];
    q.H = H;
    q.cb = cb;
    q.packed = packed;
    q.norms = norms;
    q.u_out = u_out;
    parallel_for(rows * q.G, nthreads, quant_range, &q);
    free(H);
    return 0;
}

/* ------------------------------------------------------------------------------------ */
/* Dequantise (page 1 pipeline steps 5-6: codeword times norm, inverse rotation, unpad;  */
/* H is symmetric and orthonormal, so the inverse rotation is H again).                  */
/* ------------------------------------------------------------------------------------ */

typedef struct {
    const uint8_t* packed;
    const uint16_t* norms;
    int64_t rows, cols, G;
    int g, L, fb, blk_bytes;
    const double* H;
    const double* cb;
    double* out;
} deq_ctx;

static void deq_group(const deq_ctx* d, int64_t gid, double* s, double* wh) {
    int g = d->g;
    const uint8_t* blk = d->packed + gid * d->blk_bytes;
    double n = cqo_f16_to_f64(d->norms[gid]);
    for (int i = 0; i < g; ++i) {
        int k = cqo_unpack_index(blk, d->fb, i);
        if (k >= d->L) k = d->L - 1;
        s[i] = n * d->cb[k];
    }
    for (int i = 0; i < g; ++i) {
        double acc = 0.0;
        for (int k = 0; k < g; ++k) acc += d->H[(size_t)i * g + k] * s[k];
        wh[i] = acc;
    }
}

static void deq_range(void* p, int64_t g0, int64_t g1) {
    deq_ctx* d = (deq_ctx*)p;
    double* s = (double*)malloc(sizeof(double) * (size_t)d->g);
    double* wh = (double*)malloc(sizeof(double) * (size_t)d->g);
    for (int64_t gid = g0; gid < g1; ++gid) {
        deq_group(d, gid, s, wh);
        int64_t row = gid / d->G, j = gid % d->G;
        for (int i = 0; i < d->g; ++i) {
            int64_t col = j * d->g + i;
            if (col < d->cols) d->out[row * d->cols + col] = wh[i];
        }
    }
    free(s);
    free(wh);
}

static int deq_init(deq_ctx* d, const uint8_t* packed, const uint16_t* norms, int64_t rows,
                    int64_t cols, int bits, int group_size, const float* codebook, double* cb,
                    double** H) {
    int L = cqo_levels(bits), fb = cqo_field_bits(bits);
    if (L < 0 || !is_pow2(group_size) || group_size < 8 || rows < 0 || cols < 0) return -1;
    d->packed = packed;
    d->norms = norms;
    d->rows = rows;
    d->cols = cols;
    d->G = (cols + group_size - 1) / group_size;
    d->g = group_size;
    d->L = L;
    d->fb = fb;
    d->blk_bytes = group_size * fb / 8;
    *H = (double*)malloc(sizeof(double) * (size_t)group_size * group_size);
    cqo_hadamard(group_size, *H);
    for (int k = 0; k < L; ++k) cb[k] = (double)codebook[k];
    d->H = *H;
    d->cb = cb;
    return 0;
}

int cqo_dequantize(const uint8_t* packed, const uint16_t* norms, int64_t rows, int64_t cols,
                   int bits, int group_size, const float* codebook, double* out, int nthreads) {
    deq_ctx d;
    double cb[16];
    double* H = NULL;
    if (deq_init(&d, packed, norms, rows, cols, bits, group_size, codebook, cb, &H) != 0) return -1;
    d.out = out;
    parallel_for(rows * d.G, nthreads, deq_range, &d);
    free(H);
    return 0;
}

/* ------------------------------------------------------------------------------------ */
/* GEMV, checked the slow way: dequantise each row explicitly, then a plain dot product. */
/* ------------------------------------------------------------------------------------ */

typedef struct {
    deq_ctx d;
    const void* x;
    int x_dtype, batch;
    double* y;
} gemv_ctx;

static void gemv_range(void* p, int64_t r0, int64_t r1) {
    gemv_ctx* c = (gemv_ctx*)p;
    const deq_ctx* d = &c->d;
    double* row = (double*)malloc(sizeof(double) * (size_t)(d->G * d->g));
    double* s = (double*)malloc(sizeof(double) * (size_t)d->g);
    for (int64_t r = r0; r < r1; ++r) {
        for (int64_t j = 0; j < d->G; ++j) deq_group(d, r * d->G + j, s, row + j * d->g);
        for (int b = 0; b < c->batch; ++b) {
            double acc = 0.0;
            for (int64_t col = 0; col < d->cols; ++col)
                acc += row[col] * load_elem(c->x, c->x_dtype, (int64_t)b * d->cols + col);
            c->y[(int64_t)b * d->rows + r] = acc;
        }
    }
    free(row);
    free(s);
}

int cqo_dequant_gemv(const uint8_t* packed, const uint16_t* norms, int64_t rows, int64_t cols,
                     int bits, int group_size, const float* codebook, const void* x, int x_dtype,
                     int batch, double* y, int nthreads) {
    gemv_ctx c;
    double cb[16];
    double* H = NULL;
    if (batch < 1) return -1;
    if (deq_init(&c.d, packed, norms, rows, cols, bits, group_size, codebook, cb, &H) != 0) return -1;
    c.x = x;
    c.x_dtype = x_dtype;
    c.batch = batch;
    c.y = y;
    parallel_for(rows, nthreads, gemv_range, &c);
    free(H);
    return 0;
}

/* ------------------------------------------------------------------------------------ */
/* Distortion (page 3 "Quantization Error and Accuracy Impact": relative error of the   */
/* reconstruction on random matrices).                                                   */
/* ------------------------------------------------------------------------------------ */

double cqo_rel_mse(const void* w, int dtype, const double* w_hat, int64_t n) {
    double num = 0.0, den = 0.0;
    for (int64_t i = 0; i < n; ++i) {
        double a = load_elem(w, dtype, i);
        num += (a - w_hat[i]) * (a - w_hat[i]);
        den += a * a;
    }
    return den > 0.0 ? num / den : 0.0;
}
