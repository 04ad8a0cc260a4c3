// cq_dequantize_tc.cu -- packed indices + fp16 norms -> W_hat with the inverse rotation on
// the fifth-generation tensor cores (tcgen05).
//
// Same arithmetic as cq_dequantize.cu (page "Cactus Quants CQ2-bit Quantization", "The CQ2-bit
// Implementation Pipeline" steps 5-6): w_hat = (n / sqrt(128)) H_int c[idx].  For 128 groups
// at a time the rotation is the product  D[128 groups x 128] = C[128 x 128] . H_int  (H
// symmetric), where C holds the codewords.  Each codeword, scaled by an exact power of two
// 2^cs, is split into two fp16 values hi + lo that sum to it within 2^-22 relative, so two
// fp16 MMAs with exact +-1 weights and fp32 accumulation give the fp32 result.
//
// Persistent kernel, one 448-thread CTA per SM (all 512 TMEM columns: A buffers 0-255, D
// buffers 256-511):
//   warp 0      bulk-copies each tile's packed blocks (128 groups, contiguous) into a
//               4-stage shared-memory ring;
//   warp 1      one lane issues per tile 16 tcgen05.mma (M=128, N=128, K=16): 8 for the hi
//               plane, 8 for the lo plane, A read from A buffer i % 2 in TMEM, B = H_int from
//               shared memory, into D buffer i % 2;
//   warps 2-5   decode: a thread turns its group's codes into fp16 pairs with byte permutes
//               (or a lane-held table) and writes them to the A buffer with tcgen05.st;
//   warps 6-13  two epilogue groups, one per D buffer, taking alternating tiles: a thread
//               reads its group's 128 results back, scales them by the norm and stores them.
// Decode, MMA and epilogue of consecutive tiles overlap: A and D buffers are handed over
// through their own mbarrier pairs.  One launch may cover several tensors (a job list).
//
// K order of a 2-bit group.  The MMA contracts over the 128 input elements in any order as
// long as A and B agree: column k = 16 w + 4 p + q of A holds element e = 16 w + 4 q + p, the
// code at bit 2p of byte q of packed word w, so four consecutive columns come from one
// shift + mask, and row n of the shared-memory B holds H_int[n][e(k)].
#include <algorithm>
#include <cstring>
#include <mutex>

#include "cq_device.cuh"
#include "cq_internal.h"
#include "cq_sm100.cuh"

namespace cq {
namespace {

using namespace dev;
using namespace sm100;

constexpr int kDqThreads = 64 + 128 + 256;  // producer, MMA, decode group, 2 epilogue groups
constexpr int kTile = 128;
constexpr int kStagesDq = 4;
constexpr int kACols = 128;                     // one A buffer: hi plane (64) + lo plane (64)
constexpr int kDBase = 256;                     // D buffers at columns 256 and 384
constexpr int kTmemColsDq = 512;
constexpr int kHBytes = kTile * kTile * 2;      // fp16 H_int, two 64-column swizzled halves
constexpr int kHHalf = kHBytes / 2;
constexpr uint32_t kIdescDq = idesc_f16_f32(kTile, kTile);

struct DqShape {
    long long total;   // groups
    long long cols;    // columns of W
    long long G;       // groups per row
    long long tiles;   // ceil(total / 128)
    int flat;          // cols % 128 == 0: group g's output starts at element 128 g
};

// The tensors of one launch.  Job k owns the global tiles [tile0[k], tile0[k + 1]); omap[k]
// is the output tensor map of a flat job.
template <int NJ>
struct DqJobs {
    CUtensorMap omap[NJ];  // 64-byte aligned, first
    DqShape sh[NJ];
    const uint8_t* packed[NJ];
    const uint16_t* norms[NJ];
    void* out[NJ];
    long long tile0[NJ + 1];
    int n;
};


// Job of the tiles a loop visits in increasing order: a cursor that only moves forward.
template <int NJ>
struct JobCursor {
    int k = 0;
    __device__ __forceinline__ int at(const DqJobs<NJ>& jb, long long t) {
        if constexpr (NJ > 1) {
            while (t >= jb.tile0[k + 1]) ++k;
        }
        return k;
    }
};

// Element of the group held by MMA column k.
template <int B>
__device__ __forceinline__ int elem_of_col(int k) {
    if constexpr (B == 2) {
        const int w = k >> 4, p = (k >> 2) & 3, q = k & 3;
        return 16 * w + 4 * q + p;
    } else {
        return k;
    }
}

__device__ __forceinline__ uint32_t prmt(uint32_t a, uint32_t b, uint32_t sel) {
    uint32_t d;
    asm("prmt.b32 %0, %1, %2, %3;" : "=r"(d) : "r"(a), "r"(b), "r"(sel));
    return d;
}
__device__ __forceinline__ uint32_t mad_hi(uint32_t a, uint32_t b, uint32_t c) {
    uint32_t d;
    asm("mad.hi.u32 %0, %1, %2, %3;" : "=r"(d) : "r"(a), "r"(b), "r"(c));
    return d;
}

template <bool kBF16>
__device__ __forceinline__ void store_chunk(void* out, long long elem, const float (&v)[32], int off,
                                            float scale) {
    // 8 (bf16) or 4 (fp32) consecutive values = 16 bytes
    if constexpr (kBF16) {
        uint4 o;
        o.x = pack_bf16x2(v[off + 0] * scale, v[off + 1] * scale);
        o.y = pack_bf16x2(v[off + 2] * scale, v[off + 3] * scale);
        o.z = pack_bf16x2(v[off + 4] * scale, v[off + 5] * scale);
        o.w = pack_bf16x2(v[off + 6] * scale, v[off + 7] * scale);
        st_stream16(static_cast<uint16_t*>(out) + elem, o);
    } else {
        uint4 o;
        o.x = __float_as_uint(v[off + 0] * scale);
        o.y = __float_as_uint(v[off + 1] * scale);
        o.z = __float_as_uint(v[off + 2] * scale);
        o.w = __float_as_uint(v[off + 3] * scale);
        st_stream16(static_cast<float*>(out) + elem, o);
    }
}

// Output staging for the tensor-map store: per decode group one [128 rows x 128] tile of the
// output type, as 128-byte-wide boxes of 128 rows with the 128-byte swizzle (conflict-free
// per-row writes; the TMA unit undoes the swizzle on the way out).
template <bool kBF16>
struct OutTile {
    static constexpr int kBoxes = kBF16 ? 2 : 4;        // 64 bf16 or 32 fp32 per 128-byte box
    static constexpr int kPerBox = kBF16 ? 64 : 32;
    static constexpr int kBoxBytes = kTile * 128;
    static constexpr int kBytes = kBoxes * kBoxBytes;
    // byte offset of 16-byte chunk `chunk` (of 8 bf16 / 4 fp32 values) of row m
    __device__ static int chunk_offset(int m, int chunk) {
        constexpr int kChunksPerBox = 8;
        const int box = chunk / kChunksPerBox, c = chunk % kChunksPerBox;
        return box * kBoxBytes + m * 128 + ((c ^ (m & 7)) << 4);
    }
};

template <int B, int L, bool kBF16, int NJ>
__global__ void __launch_bounds__(kDqThreads, 1)
    dequantize_tc_kernel(const __grid_constant__ DqJobs<NJ> jobs, const float* __restrict__ codebook,
                         unsigned* __restrict__ status) {
    extern __shared__ uint8_t smem_raw[];
    __shared__ __align__(8) uint64_t full_bar[kStagesDq], empty_bar[kStagesDq];
    __shared__ __align__(8) uint64_t afull_bar[2], aempty_bar[2], dfull_bar[2], dempty_bar[2];
    __shared__ uint32_t tmem_slot;
    __shared__ uint32_t tab_s[16];  // fp16 (hi | lo << 16) of every code (3- and 4-bit codes)
    // norms handed from decode to epilogue, slot i % 4: decode of tile i + 4 waits (through
    // the MMA of tile i + 2) until the epilogue of tile i has released its D buffer
    __shared__ float norm_s[4][kTile];
    constexpr int kCodeBytes = kTile * 16 * B;
    constexpr int kStageBytes = kCodeBytes + kTile * 2;  // codes, then the tile's fp16 norms

    uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
    uint8_t* hmat = smem;
    uint8_t* ring = smem + kHBytes;
    uint8_t* stage_out = ring + kStagesDq * kStageBytes;  // 2 x OutTile (1024-aligned)
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const long long ntiles = jobs.tile0[jobs.n];

    pdl_trigger();


    // B operand: row n, column k = H_int[n][e(k)] (fp16 +-1), K-major, 128-byte swizzle
    for (int item = threadIdx.x; item < kTile * 16; item += kDqThreads) {
        const int n = item >> 4, c16 = item & 15;
        uint32_t w4[4];
#pragma unroll
        for (int p = 0; p < 4; ++p) {
            const int k0 = c16 * 8 + 2 * p;
            const uint32_t lo = (__popc(n & elem_of_col<B>(k0)) & 1) ? 0xBC00u : 0x3C00u;
            const uint32_t hi = (__popc(n & elem_of_col<B>(k0 + 1)) & 1) ? 0xBC00u : 0x3C00u;
            w4[p] = lo | (hi << 16);
        }
        const int half = c16 >> 3, kl = (c16 & 7);
        *reinterpret_cast<uint4*>(hmat + half * kHHalf + n * 128 + ((kl ^ (n & 7)) << 4)) =
            make_uint4(w4[0], w4[1], w4[2], w4[3]);
    }
    fence_proxy_async_smem();

    if (threadIdx.x == 0) {
        for (int s = 0; s < kStagesDq; ++s) {
            mbar_init(&full_bar[s], 1);
            mbar_init(&empty_bar[s], 4);
        }
        for (int a = 0; a < 2; ++a) {
            mbar_init(&afull_bar[a], 4);   // the decode group's four warps
            mbar_init(&aempty_bar[a], 1);  // MMA completion
            mbar_init(&dfull_bar[a], 1);   // MMA completion
            mbar_init(&dempty_bar[a], 4);  // epilogue group a's four warps
        }
        fence_mbar_init();
        // the first tiles' codes and norms of this CTA into L2 while the previous kernel finishes
        long long t = blockIdx.x;
        JobCursor<NJ> cur;
        for (int i = 0; i < kStagesDq && t < ntiles; ++i, t += gridDim.x) {
            const int k = cur.at(jobs, t);
            const DqShape& sh = jobs.sh[k];
            const long long g0 = (t - jobs.tile0[k]) * kTile;
            const long long n = sh.total - g0 < kTile ? sh.total - g0 : kTile;
            bulk_prefetch_l2(jobs.packed[k] + g0 * (16 * B), static_cast<uint32_t>(n) * (16 * B));
            if (n == kTile) bulk_prefetch_l2(jobs.norms[k] + g0, kTile * 2);
        }
    }
    if (warp == 1) tmem_alloc(&tmem_slot, kTmemColsDq);
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tbase = tmem_slot;
    pdl_wait();  // on-chip set-up above; global memory only from here

    // codewords c_k 2^cs = hi_k + lo_k in fp16
    float cmax = 0.0f;
#pragma unroll
    for (int k = 0; k < L; ++k) cmax = fmaxf(cmax, fabsf(__ldg(codebook + k)));
    const int cs = (cmax > 0.0f) ? (13 - ilogbf(cmax)) : 0;
    uint32_t hl[4], hh[4], ll[4], lh[4];  // bytes of hi / lo for codes 0..3
    uint32_t th_lo = 0, th_hi = 0, tl_lo = 0, tl_hi = 0;
#pragma unroll
    for (int k = 0; k < 4; ++k) {
        const float x = ldexpf(__ldg(codebook + (k < L ? k : L - 1)), cs);
        const __half h = __float2half_rn(x);
        const __half l = __float2half_rn(x - __half2float(h));
        hl[k] = __half_as_ushort(h) & 0xffu;
        hh[k] = __half_as_ushort(h) >> 8;
        ll[k] = __half_as_ushort(l) & 0xffu;
        lh[k] = __half_as_ushort(l) >> 8;
        th_lo |= hl[k] << (8 * k);
        th_hi |= hh[k] << (8 * k);
        tl_lo |= ll[k] << (8 * k);
        tl_hi |= lh[k] << (8 * k);
    }
    if (threadIdx.x < 16) {
        const float x = ldexpf(__ldg(codebook + (threadIdx.x < L ? threadIdx.x : L - 1)), cs);
        const __half h = __float2half_rn(x);
        const __half l = __float2half_rn(x - __half2float(h));
        tab_s[threadIdx.x] = static_cast<uint32_t>(__half_as_ushort(h)) |
                             (static_cast<uint32_t>(__half_as_ushort(l)) << 16);
    }
    const float inv_scale = ldexpf(1.0f, -cs) * kInvSqrt128;
    __syncthreads();  // tab_s
    // the same table held one entry per lane, repeated every 2^B lanes, so that a shuffle whose
    // index is the code plus any higher bits (only the low 5 bits of the index count) reads it
    const uint32_t tab_lane = tab_s[lane & ((1 << B) - 1) & 15];

    if (warp == 0) {
        // ---------------- bulk-copy producer ----------------
        if (lane == 0) {
            int i = 0;
            JobCursor<NJ> cur;
            for (long long t = blockIdx.x; t < ntiles; t += gridDim.x, ++i) {
                const int st = i % kStagesDq;
                if (!mbar_wait(&empty_bar[st], ((i / kStagesDq) & 1) ^ 1, status)) break;
                const int k = cur.at(jobs, t);
                const DqShape& sh = jobs.sh[k];
                const long long g0 = (t - jobs.tile0[k]) * kTile;
                const long long n = sh.total - g0 < kTile ? sh.total - g0 : kTile;
                const uint32_t bytes = static_cast<uint32_t>(n) * (16 * B);
                // full tiles bring their 256 bytes of norms along (16-byte aligned: the norms
                // array starts on 16 bytes and a tile's norms start at 256 * tile)
                const bool nrm_bulk = n == kTile;
                mbar_arrive_expect_tx(&full_bar[st], bytes + (nrm_bulk ? kTile * 2 : 0));
                bulk_load(ring + st * kStageBytes, jobs.packed[k] + g0 * (16 * B), bytes, &full_bar[st]);
                if (nrm_bulk) bulk_load(ring + st * kStageBytes + kCodeBytes, jobs.norms[k] + g0, kTile * 2, &full_bar[st]);
            }
            for (int k = 0; k < kStagesDq && k < i; ++k) {
                const int ii = i - 1 - k;
                mbar_wait(&empty_bar[ii % kStagesDq], (ii / kStagesDq) & 1, status);
            }
        }
    } else if (warp == 1) {
        // ---------------- MMA issuer ----------------
        if (lane == 0) {
            int i = 0;
            for (long long t = blockIdx.x; t < ntiles; t += gridDim.x, ++i) {
                const int e = i & 1;  // A buffer and D buffer of this tile
                if (!mbar_wait(&afull_bar[e], (i >> 1) & 1, status)) break;
                if (!mbar_wait(&dempty_bar[e], ((i >> 1) & 1) ^ 1, status)) break;
                tc_fence_after();
                const uint32_t a_hi = tbase + e * kACols, a_lo = a_hi + 64, d = tbase + kDBase + e * kTile;
                const uint32_t b_base = smem_u32(hmat);
#pragma unroll
                for (int k = 0; k < kTile / 16; ++k)
                    mma_f16_tmem_a(d, a_hi + 8 * k,
                                   smem_desc_sw128(b_base + (k >> 2) * kHHalf + (k & 3) * 32), kIdescDq,
                                   k > 0);
#pragma unroll
                for (int k = 0; k < kTile / 16; ++k)
                    mma_f16_tmem_a(d, a_lo + 8 * k,
                                   smem_desc_sw128(b_base + (k >> 2) * kHHalf + (k & 3) * 32), kIdescDq,
                                   true);
                mma_commit(&aempty_bar[e]);
                mma_commit(&dfull_bar[e]);
            }
        }
    } else if (warp < 6) {
        // ---------------- decode: codes -> A buffer (i & 1) ----------------
        const int quad = warp & 3;
        const int m = quad * 32 + lane;
        const uint32_t lane_off = static_cast<uint32_t>(quad * 32) << 16;
        int i = 0;
        JobCursor<NJ> cur;
        for (long long t = blockIdx.x; t < ntiles; t += gridDim.x, ++i) {
            const int k = cur.at(jobs, t);
            const DqShape& sh = jobs.sh[k];
            const long long tl = t - jobs.tile0[k];
            const int st = i % kStagesDq;
            const int e = i & 1;
            bool ok = mbar_wait(&full_bar[st], (i / kStagesDq) & 1, status);
            ok = ok && mbar_wait(&aempty_bar[e], ((i >> 1) & 1) ^ 1, status);
            // the group's four warps decide together whether to go on
            if (!named_barrier_and(1, 128, ok)) break;
            tc_fence_after();
            const uint32_t a_hi = tbase + lane_off + e * kACols, a_lo = a_hi + 64;
            const long long gid = tl * kTile + m;
            const bool valid = gid < sh.total;
            {
                // this group's norm for the epilogue (full tiles: from the stage; the last,
                // partial tile: from global memory)
                const bool full_tile = sh.total - tl * kTile >= kTile;
                const uint16_t* nstage = reinterpret_cast<const uint16_t*>(ring + st * kStageBytes + kCodeBytes);
                const uint16_t hb = full_tile ? nstage[m] : (valid ? __ldg(jobs.norms[k] + gid) : uint16_t(0));
                norm_s[i & 3][m] = __half2float(__ushort_as_half(hb));
            }
            uint32_t wd[4 * B];
            {
                const uint4* src = reinterpret_cast<const uint4*>(ring + st * kStageBytes + m * (16 * B));
#pragma unroll
                for (int v = 0; v < B; ++v) {
                    const uint4 u = valid ? src[v] : make_uint4(0, 0, 0, 0);
                    wd[4 * v + 0] = u.x;
                    wd[4 * v + 1] = u.y;
                    wd[4 * v + 2] = u.z;
                    wd[4 * v + 3] = u.w;
                }
            }

            // A planes: 64 columns each, written 32 at a time
#pragma unroll
            for (int half = 0; half < 2; ++half) {
                uint32_t rh[32], rl[32];
                if constexpr (B == 2) {
#pragma unroll
                    for (int ww = 0; ww < 4; ++ww) {
                        const uint32_t word = wd[4 * half + ww];
#pragma unroll
                        for (int p = 0; p < 4; ++p) {
                            const uint32_t sw = (word >> (2 * p)) & 0x03030303u;
                            const uint32_t s0 = sw * 0x11u + 0x4040u;
                            const uint32_t s1 = mad_hi(sw, 0x110000u, 0x4040u);
                            const int col = 8 * ww + 2 * p;  // within this 32-column half
                            rh[col] = prmt(th_lo, th_hi, s0);
                            rh[col + 1] = prmt(th_lo, th_hi, s1);
                            rl[col] = prmt(tl_lo, tl_hi, s0);
                            rl[col + 1] = prmt(tl_lo, tl_hi, s1);
                        }
                    }
                } else {
                    static_assert(L == (1 << B), "3/4-bit codebooks use every code");
#pragma unroll
                    for (int c = 0; c < 32; ++c) {
                        const int e0 = 64 * half + 2 * c;  // elements e0, e0 + 1
                        uint32_t t[2];
#pragma unroll
                        for (int u = 0; u < 2; ++u) {
                            // the code sits in the low B bits; bits above it are ignored by the
                            // lane-repeated table
                            const int bit = B * (e0 + u);
                            const uint32_t lo = wd[bit >> 5];
                            uint32_t idx;
                            if ((bit & 31) + B <= 32) {
                                idx = lo >> (bit & 31);
                            } else {
                                idx = __funnelshift_r(lo, wd[(bit >> 5) + 1], bit & 31);
                            }
                            t[u] = __shfl_sync(kFullMask, tab_lane, static_cast<int>(idx));
                        }
                        rh[c] = prmt(t[0], t[1], 0x5410u);
                        rl[c] = prmt(t[0], t[1], 0x7632u);
                    }
                }
                tmem_st32(a_hi + 32 * half, rh);
                tmem_st32(a_lo + 32 * half, rl);
            }
            tmem_st_wait();
            tc_fence_before();
            // the stage's words are consumed; order these generic reads before the producer's
            // next bulk write into the stage
            fence_proxy_async_smem();
            __syncwarp();
            if (lane == 0) {
                mbar_arrive(&empty_bar[st]);
                mbar_arrive(&afull_bar[e]);
            }
        }
    } else {
        // ---------------- epilogue group e: D buffer e -> W_hat (tiles i = e mod 2) ----------
        const int e = (warp - 6) >> 2;
        const int quad = warp & 3;
        const int m = quad * 32 + lane;
        const uint32_t lane_off = static_cast<uint32_t>(quad * 32) << 16;
        const uint32_t d = tbase + lane_off + kDBase + e * kTile;
        const bool leader = (warp == 6 + 4 * e) && lane == 0;
        int i = e;
        JobCursor<NJ> cur;
        for (long long t = blockIdx.x + static_cast<long long>(e) * gridDim.x; t < ntiles;
             t += 2LL * gridDim.x, i += 2) {
            const int k = cur.at(jobs, t);
            const DqShape& sh = jobs.sh[k];
            const long long tl = t - jobs.tile0[k];
            const long long gid = tl * kTile + m;
            const bool valid = gid < sh.total;
            bool ok = mbar_wait(&dfull_bar[e], (i >> 1) & 1, status);
            // before the staging tile is rewritten, this group's previous stores have read it
            if (sh.flat && leader) bulk_wait_read0();
            if (!named_barrier_and(2 + e, 128, ok)) break;
            tc_fence_after();
            const float scale = norm_s[i & 3][m] * inv_scale;
            constexpr int kPer = kBF16 ? 8 : 4;  // values per 16-byte chunk
            if (sh.flat) {
                // stage the tile in shared memory, then one tensor-map store per box
                uint8_t* so = stage_out + e * OutTile<kBF16>::kBytes;
#pragma unroll
                for (int c = 0; c < kTile / 32; ++c) {
                    float v[32];
                    tmem_ld32(d + 32 * c, v);
                    tmem_ld_wait();
#pragma unroll
                    for (int q = 0; q < 32 / kPer; ++q) {
                        const int off = q * kPer;
                        uint4 o;
                        if constexpr (kBF16) {
                            o.x = pack_bf16x2(v[off + 0] * scale, v[off + 1] * scale);
                            o.y = pack_bf16x2(v[off + 2] * scale, v[off + 3] * scale);
                            o.z = pack_bf16x2(v[off + 4] * scale, v[off + 5] * scale);
                            o.w = pack_bf16x2(v[off + 6] * scale, v[off + 7] * scale);
                        } else {
                            o.x = __float_as_uint(v[off + 0] * scale);
                            o.y = __float_as_uint(v[off + 1] * scale);
                            o.z = __float_as_uint(v[off + 2] * scale);
                            o.w = __float_as_uint(v[off + 3] * scale);
                        }
                        *reinterpret_cast<uint4*>(so + OutTile<kBF16>::chunk_offset(m, (32 * c + off) / kPer)) = o;
                    }
                }
                // D buffer read out: the MMAs of the tile after next may overwrite it
                tc_fence_before();
                __syncwarp();
                if (lane == 0) mbar_arrive(&dempty_bar[e]);
                fence_proxy_async_smem();
                named_barrier(2 + e, 128);
                if (leader) {
#pragma unroll
                    for (int b = 0; b < OutTile<kBF16>::kBoxes; ++b)
                        tma_store_2d(&jobs.omap[k], b * OutTile<kBF16>::kPerBox, static_cast<int>(tl * kTile),
                                     so + b * OutTile<kBF16>::kBoxBytes);
                    bulk_commit();
                }
            } else {
                const long long row = gid / sh.G, j = gid - (gid / sh.G) * sh.G;
                const long long base = row * sh.cols + j * kTile;
#pragma unroll
                for (int c = 0; c < kTile / 32; ++c) {
                    float v[32];
                    tmem_ld32(d + 32 * c, v);
                    tmem_ld_wait();
                    if (!valid) continue;
#pragma unroll
                    for (int q = 0; q < 32 / kPer; ++q) {
                        const int off = q * kPer;
                        if (j * kTile + 32 * c + off < sh.cols)
                            store_chunk<kBF16>(jobs.out[k], base + 32 * c + off, v, off, scale);
                    }
                }
                tc_fence_before();
                __syncwarp();
                if (lane == 0) mbar_arrive(&dempty_bar[e]);
            }
        }
        if (leader) bulk_wait0();  // tensor-map stores done before exit
    }

    tc_fence_before();
    __syncthreads();
    if (warp == 1) {
        tc_fence_after();
        tmem_dealloc(tbase, kTmemColsDq);
    }
}

template <int B, int L, bool kBF16, int NJ>
cudaError_t launch_dq(const DqJobs<NJ>& jobs, const float* cb, unsigned* status, cudaStream_t st) {
    // at least 120 KB so that two CTAs never share an SM: each takes all 512 TMEM columns, and
    // with programmatic launch a CTA of the next kernel could otherwise wait inside
    // tcgen05.alloc until the previous one frees them
    const int smem = std::max(kHBytes + kStagesDq * (kTile * 16 * B + kTile * 2) + 2 * OutTile<kBF16>::kBytes + 1024,
                              120 * 1024);
    int dev = 0;
    cudaError_t e = cudaGetDevice(&dev);
    if (e != cudaSuccess) return e;
    static unsigned long long configured = 0;  // one bit per device
    const unsigned long long bit = 1ull << (dev & 63);
    if (!(configured & bit)) {
        e = cudaFuncSetAttribute(dequantize_tc_kernel<B, L, kBF16, NJ>, cudaFuncAttributeMaxDynamicSharedMemorySize, smem);
        if (e != cudaSuccess) return e;
        configured |= bit;
    }
    const long long ntiles = jobs.tile0[jobs.n];
    const int grid = static_cast<int>(std::max<long long>(1, std::min<long long>(ntiles, sm_count())));
    return launch_pdl(dequantize_tc_kernel<B, L, kBF16, NJ>, dim3(grid), dim3(kDqThreads), smem, st,
                      jobs, cb, status);
}

// Shape, outputs and (flat shapes) the output tensor map of one tensor as job k of `jobs`.
template <int NJ>
bool add_job(DqJobs<NJ>& jobs, int k, const uint8_t* packed, const uint16_t* norms,
             const Shape& sh, void* out, bool bf16) {
    DqShape ds;
    ds.total = sh.total_groups;
    ds.cols = sh.cols;
    ds.G = sh.groups_per_row;
    ds.tiles = (sh.total_groups + kTile - 1) / kTile;
    ds.flat = sh.cols % kTile == 0;
    std::memset(&jobs.omap[k], 0, sizeof(CUtensorMap));
    if (ds.flat) {
        // the output viewed as [groups x 128] values, boxes of 128 bytes x 128 rows
        const cuuint64_t gdim[2] = {static_cast<cuuint64_t>(kTile), static_cast<cuuint64_t>(ds.total)};
        const cuuint64_t gstride[1] = {static_cast<cuuint64_t>(kTile) * (bf16 ? 2 : 4)};
        const cuuint32_t box[2] = {static_cast<cuuint32_t>(bf16 ? OutTile<true>::kPerBox : OutTile<false>::kPerBox), kTile};
        const cuuint32_t estride[2] = {1, 1};
        EncodeTiledFn enc = tensor_map_encoder();
        if (enc == nullptr) return false;
        const CUresult r = enc(&jobs.omap[k], bf16 ? CU_TENSOR_MAP_DATA_TYPE_BFLOAT16 : CU_TENSOR_MAP_DATA_TYPE_FLOAT32,
                               2, out, gdim, gstride, box, estride, CU_TENSOR_MAP_INTERLEAVE_NONE,
                               CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_NONE,
                               CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
        if (r != CUDA_SUCCESS) return false;
    }
    jobs.sh[k] = ds;
    jobs.packed[k] = packed;
    jobs.norms[k] = norms;
    jobs.out[k] = out;
    jobs.tile0[k + 1] = jobs.tile0[k] + ds.tiles;
    return true;
}

template <int NJ>
cudaError_t launch_bits(int bits, int out_dtype, const DqJobs<NJ>& jobs, const float* cb,
                        unsigned* status, cudaStream_t st) {
    const bool bf = out_dtype == CQ_BF16;
    switch (bits) {
        case CQ_BITS_TERNARY:
            return bf ? launch_dq<2, 3, true, NJ>(jobs, cb, status, st) : launch_dq<2, 3, false, NJ>(jobs, cb, status, st);
        case 2:
            return bf ? launch_dq<2, 4, true, NJ>(jobs, cb, status, st) : launch_dq<2, 4, false, NJ>(jobs, cb, status, st);
        case 3:
            return bf ? launch_dq<3, 8, true, NJ>(jobs, cb, status, st) : launch_dq<3, 8, false, NJ>(jobs, cb, status, st);
        default:
            return bf ? launch_dq<4, 16, true, NJ>(jobs, cb, status, st) : launch_dq<4, 16, false, NJ>(jobs, cb, status, st);
    }
}

// Jobs per batched launch: the job list travels in the kernel parameters (at most 32 KB).
constexpr int kBatchJobs = 128;
static_assert(sizeof(DqJobs<kBatchJobs>) < 32000, "kernel parameter space");

}  // namespace

bool dequantize_tc_supported(int out_dtype, const Shape& sh) {
    if (sh.cols % (out_dtype == CQ_BF16 ? 8 : 4) != 0) return false;
    if (sh.cols % kTile == 0 && (sh.total_groups >= (1LL << 31) || tensor_map_encoder() == nullptr)) return false;
    return true;
}

cudaError_t launch_dequantize_tc(const uint8_t* packed, const uint16_t* norms, const Shape& sh,
                                 int bits, const float* codebook, void* out, int out_dtype,
                                 unsigned* status, cudaStream_t stream) {
    DqJobs<1> jobs;
    jobs.n = 1;
    jobs.tile0[0] = 0;
    if (!add_job(jobs, 0, packed, norms, sh, out, out_dtype == CQ_BF16)) return cudaErrorInvalidValue;
    return launch_bits(bits, out_dtype, jobs, codebook, status, stream);
}

cudaError_t launch_dequantize_tc_batch(const DequantizeItem* items, int count, int bits,
                                       const float* codebook, int out_dtype, unsigned* status,
                                       cudaStream_t stream) {
    static DqJobs<kBatchJobs> jobs;  // host staging (large); calls are serialised below
    static std::mutex mu;
    std::lock_guard<std::mutex> lock(mu);
    for (int i0 = 0; i0 < count; i0 += kBatchJobs) {
        const int n = std::min(kBatchJobs, count - i0);
        jobs.n = n;
        jobs.tile0[0] = 0;
        for (int k = 0; k < n; ++k) {
            const DequantizeItem& it = items[i0 + k];
            if (!add_job(jobs, k, it.packed, it.norms, it.sh, it.out, out_dtype == CQ_BF16))
                return cudaErrorInvalidValue;
        }
        const cudaError_t e = launch_bits(bits, out_dtype, jobs, codebook, status, stream);
        if (e != cudaSuccess) return e;
    }
    return cudaSuccess;
}

}  // namespace cq
