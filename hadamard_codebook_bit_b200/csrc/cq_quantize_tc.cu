// cq_quantize_tc.cu -- bf16 W -> packed indices + fp16 norms with the rotation on the
// fifth-generation tensor cores (tcgen05), for bf16 inputs whose rows start on 16 bytes.
//
// Same arithmetic as cq_quantize.cu (page "Cactus Quants CQ2-bit Quantization", "The CQ2-bit
// Implementation Pipeline" steps 1-4): the rotation r = H_int v of 128 groups at a time is
// the product  R[128 groups x 128] = V[128 x 128] . H_int[128 x 128]  (H symmetric), a bf16 x
// bf16 MMA with exact +-1 weights and fp32 accumulation, which is how the pages write the
// rotation ("rot @ H", page "How CQ2-bit Quantization Contributes to Needle 2's Small
// Footprint", "Hadamard Rotation").
//
// Persistent kernel, one 576-thread CTA per SM:
//   warp 0      TMA producer: 128 x 128 bf16 tiles (two 64-column boxes, 128-byte swizzle)
//               into a 4-stage shared-memory ring;
//   warp 1      owns 512 TMEM columns; one lane issues 8 tcgen05.mma (M=128, N=128, K=16)
//               per tile into one of four TMEM accumulators, then commits to the stage's
//               "empty" barrier and the accumulator's "full" barrier;
//   warps 2-17  four epilogue groups of four warps (one per TMEM lane quadrant) take tiles in
//               turn: each thread reads its group's 128 rotated values from TMEM, forms the
//               norm, the thresholds m_k * ||r||, the indices, and stores the packed block and
//               the fp16 norm.
// One launch may cover several tensors (a job list in the kernel parameters): the tiles of
// all jobs form one index space that the CTAs stride through.
// H_int lives in shared memory in the same swizzled K-major layout (built once per CTA).
//
// Tile -> groups: the tensor map views W as [R_eff rows x C_eff cols]; tile (rb, j) covers
// rows 128 rb .. 128 rb + 127 and columns 128 j .. 128 j + 127 (zero filled past the edges,
// which is the pages' zero padding); its lane m is group (128 rb + m) * G_eff + j.  With
// cols % 128 == 0 the whole matrix is viewed as [groups x 128] (G_eff = 1), so one tile is
// 128 consecutive groups and the packed output of a tile is one contiguous block.
#include <algorithm>
#include <cmath>
#include <cstring>
#include <mutex>

#include "cq_device.cuh"
#include "cq_internal.h"
#include "cq_sm100.cuh"

namespace cq {
namespace {

using namespace dev;
using namespace sm100;

constexpr int kEpiGroups = 4;                          // epilogue warpgroups = TMEM accumulators
constexpr int kTcThreads = 64 + 128 * kEpiGroups;      // producer + MMA warps, then epilogue
constexpr int kTile = 128;                 // groups per tile (MMA M) = elements per group (K, N)
constexpr int kStagesTc = 4;
constexpr int kTileBytes = kTile * kTile * 2;  // 32 KiB of bf16
constexpr int kHalfBytes = kTileBytes / 2;     // one 64-column box
constexpr int kTmemCols = 128 * kEpiGroups;    // one fp32 accumulator of 128 columns per group
constexpr uint32_t kIdesc = idesc_bf16_f32(kTile, kTile);

struct TcShape {
    long long r_eff, g_eff, tiles_r, tiles;
};

// The tensors of one launch.  Job k owns the global tiles [tile0[k], tile0[k + 1]).
template <int NJ>
struct TcJobs {
    CUtensorMap map[NJ];  // 64-byte aligned, first
    TcShape sh[NJ];
    uint8_t* packed[NJ];
    uint16_t* norms[NJ];
    long long tile0[NJ + 1];
    int n;
};


// Job of the tiles a loop visits in increasing order: a cursor that only moves forward.
template <int NJ>
struct JobCursor {
    int k = 0;
    __device__ __forceinline__ int at(const TcJobs<NJ>& jb, long long t) {
        if constexpr (NJ > 1) {
            while (t >= jb.tile0[k + 1]) ++k;
        }
        return k;
    }
};

// Byte offset of element (row, k) of a 128 x 128 bf16 K-major tile stored as two 64-column
// halves, each with the 128-byte swizzle (16-byte chunk index XOR row % 8).
__device__ __forceinline__ int sw128_offset(int row, int k) {
    const int half = k >> 6, kl = k & 63;
    return half * kHalfBytes + row * 128 + (((kl >> 3) ^ (row & 7)) << 4) + (kl & 7) * 2;
}

// --- 2-bit / ternary packing by sign bits -------------------------------------------------
// With sorted thresholds T_0 < T_1 (< T_2), s_k = [r > T_k] is the sign bit of e_k = T_k - r
// (rounding never flips a sign; r == T_k gives +0, i.e. "not greater", the tie going low),
// and the index sum_k s_k has bits  b1 = s_1,  b0 = s_0 ^ s_1 (^ s_2).  The subtractions run
// two elements at a time on the FMA pipe (f32x2); the bits are appended into the packed word
// with funnel shifts, top element first, so element i lands at bits 2i, 2i+1.

__device__ __forceinline__ uint64_t f2pack(float a, float b) {
    uint64_t r;
    asm("mov.b64 %0, {%1, %2};" : "=l"(r) : "f"(a), "f"(b));
    return r;
}
__device__ __forceinline__ void f2unpack(uint64_t p, uint32_t& lo, uint32_t& hi) {
    asm("mov.b64 {%0, %1}, %2;" : "=r"(lo), "=r"(hi) : "l"(p));
}
__device__ __forceinline__ uint64_t f2sub(uint64_t a, uint64_t b) {
    uint64_t r;
    asm("sub.rn.f32x2 %0, %1, %2;" : "=l"(r) : "l"(a), "l"(b));
    return r;
}

// v[OFF .. OFF+15] -> one word of 16 two-bit codes; pairs (2i, 2i+1) share one f32x2
// subtraction.
template <int L, int OFF>
__device__ __forceinline__ uint32_t pack2_signbits(const float (&v)[32], const float (&T)[L - 1]) {
    static_assert(L == 3 || L == 4, "2-bit fields");
    uint64_t tp[L - 1];
#pragma unroll
    for (int k = 0; k < L - 1; ++k) tp[k] = f2pack(T[k], T[k]);
    uint32_t w = 0u;
#pragma unroll
    for (int i = 7; i >= 0; --i) {
        const uint64_t r = f2pack(v[OFF + 2 * i], v[OFF + 2 * i + 1]);
        uint32_t e0x, e0y, e1x, e1y;
        f2unpack(f2sub(tp[0], r), e0x, e0y);
        f2unpack(f2sub(tp[1], r), e1x, e1y);
        uint32_t lx = e0x ^ e1x, ly = e0y ^ e1y;
        if constexpr (L == 4) {
            uint32_t e2x, e2y;
            f2unpack(f2sub(tp[2], r), e2x, e2y);
            lx ^= e2x;
            ly ^= e2y;
        }
        w = __funnelshift_l(e1y, w, 1);  // element 2i+1: b1, b0
        w = __funnelshift_l(ly, w, 1);
        w = __funnelshift_l(e1x, w, 1);  // element 2i: b1, b0
        w = __funnelshift_l(lx, w, 1);
    }
    return w;
}

// --- 3/4-bit nearest codeword through a warp-held bucket table ---------------------------
// In normalised units u = r / n the decision thresholds are the fixed codebook midpoints m_k.
// u is mapped monotonically onto 32 buckets (t = sat(u sA + 1/2), bucket = rint(31 t)); lane b
// holds bucket b's entry: the bits of the one midpoint falling in that bucket (or a huge
// finite value) with the number of midpoints below the bucket in the low 4 mantissa bits.  The
// index is then  base + [u > threshold]  after one shuffle.  Clearing the low mantissa bits
// moves a threshold by at most 15 ulp, far inside the 1e-5 decision tolerance.  If a bucket
// would hold two midpoints (a crowded custom codebook) the select tree is used instead.
struct BucketLookup {
    uint32_t entry;
    float sA;
    bool ok;
};

__device__ __forceinline__ uint32_t bucket_of(float u, float sA) {
    const float t = __saturatef(fmaf(u, sA, 0.5f));
    return __float_as_uint(fmaf(t, 31.0f, 12582912.0f)) & 31u;  // 1.5 * 2^23: rint in the low bits
}

template <int L>
__device__ __forceinline__ BucketLookup make_buckets(const float (&mid)[L - 1], int lane) {
    BucketLookup bl;
    float span = fmaxf(fabsf(mid[0]), fabsf(mid[L - 2])) * 1.1f;
    if (!(span > 0.0f)) span = 1.0f;
    bl.sA = 0.5f / span;
    uint32_t thr = 0x7f7ffff0u, base = 0u;
    int cnt = 0;
#pragma unroll
    for (int k = 0; k < L - 1; ++k) {
        const uint32_t b = bucket_of(mid[k], bl.sA);
        if (b < static_cast<uint32_t>(lane)) {
            ++base;
        } else if (b == static_cast<uint32_t>(lane)) {
            thr = __float_as_uint(mid[k]) & ~15u;
            ++cnt;
        }
    }
    bl.entry = thr | base;
    bl.ok = !__any_sync(kFullMask, cnt > 1);
    return bl;
}

__device__ __forceinline__ uint32_t bucket_index(float u, const BucketLookup& bl) {
    const uint32_t e = __shfl_sync(kFullMask, bl.entry, static_cast<int>(bucket_of(u, bl.sA)));
    return (e & 15u) + (u > __uint_as_float(e) ? 1u : 0u);
}

// kChecked: the codebook may crowd a bucket, so the kernel checks and keeps the select tree
// as a fallback; without it (a codebook checked on the host) only the bucket search is built.
template <int B, int L, int NJ, bool kChecked>
__global__ void __launch_bounds__(kTcThreads, 1)
    quantize_tc_kernel(const __grid_constant__ TcJobs<NJ> jobs, const float* __restrict__ codebook,
                       unsigned* __restrict__ status) {
    extern __shared__ uint8_t smem_raw[];
    __shared__ __align__(8) uint64_t full_bar[kStagesTc], empty_bar[kStagesTc];
    __shared__ __align__(8) uint64_t tfull_bar[kEpiGroups], tempty_bar[kEpiGroups];
    __shared__ uint32_t tmem_slot;

    // 1024-byte aligned region: H_int, then the stage ring
    uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
    uint8_t* hmat = smem;
    uint8_t* ring = smem + kTileBytes;

    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const long long ntiles = jobs.tile0[jobs.n];
    pdl_trigger();

    // H_int (+1 = 0x3F80, -1 = 0xBF80 in bf16), row n = output element, column k = input element
    for (int item = threadIdx.x; item < kTile * 16; item += kTcThreads) {
        const int n = item >> 4, c16 = item & 15;  // 16 chunks of 8 elements per row
        uint32_t w4[4];
#pragma unroll
        for (int p = 0; p < 4; ++p) {
            const int k0 = c16 * 8 + 2 * p;
            const uint32_t lo = (__popc(n & k0) & 1) ? 0xBF80u : 0x3F80u;
            const uint32_t hi = (__popc(n & (k0 + 1)) & 1) ? 0xBF80u : 0x3F80u;
            w4[p] = lo | (hi << 16);
        }
        *reinterpret_cast<uint4*>(hmat + sw128_offset(n, c16 * 8)) = make_uint4(w4[0], w4[1], w4[2], w4[3]);
    }
    fence_proxy_async_smem();

    if (threadIdx.x == 0) {
        for (int s = 0; s < kStagesTc; ++s) {
            mbar_init(&full_bar[s], 1);
            mbar_init(&empty_bar[s], 1);
        }
        for (int a = 0; a < kEpiGroups; ++a) {
            mbar_init(&tfull_bar[a], 1);
            mbar_init(&tempty_bar[a], 4);
        }
        fence_mbar_init();
        // the first tiles of this CTA into L2 while the previous kernel finishes
        long long t = blockIdx.x;
        JobCursor<NJ> cur;
        for (int i = 0; i < kStagesTc && t < ntiles; ++i, t += gridDim.x) {
            const int k = cur.at(jobs, t);
            const TcShape& sh = jobs.sh[k];
            const long long tl = t - jobs.tile0[k];
            const int rb = static_cast<int>(tl % sh.tiles_r), j = static_cast<int>(tl / sh.tiles_r);
            tma_prefetch_2d(&jobs.map[k], kTile * j, kTile * rb);
            tma_prefetch_2d(&jobs.map[k], kTile * j + 64, kTile * rb);
        }
    }
    if (warp == 1) tmem_alloc(&tmem_slot, kTmemCols);
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tbase = tmem_slot;
    pdl_wait();  // on-chip set-up above; global memory only from here

    if (warp == 0) {
        // ---------------- TMA producer ----------------
        if (lane == 0) {
            int i = 0;
            JobCursor<NJ> cur;
            for (long long t = blockIdx.x; t < ntiles; t += gridDim.x, ++i) {
                const int st = i % kStagesTc;
                const uint32_t ph = (i / kStagesTc) & 1;
                if (!mbar_wait(&empty_bar[st], ph ^ 1, status)) break;
                const int k = cur.at(jobs, t);
                const TcShape& sh = jobs.sh[k];
                const long long tl = t - jobs.tile0[k];
                const int rb = static_cast<int>(tl % sh.tiles_r);
                const int j = static_cast<int>(tl / sh.tiles_r);
                uint8_t* dst = ring + st * kTileBytes;
                mbar_arrive_expect_tx(&full_bar[st], kTileBytes);
                tma_load_2d(dst, &jobs.map[k], kTile * j, kTile * rb, &full_bar[st]);
                tma_load_2d(dst + kHalfBytes, &jobs.map[k], kTile * j + 64, kTile * rb, &full_bar[st]);
            }
            // drain: wait (bounded) until every stage this CTA filled has been consumed
            for (int k = 0; k < kStagesTc && k < i; ++k) {
                const int ii = i - 1 - k;
                mbar_wait(&empty_bar[ii % kStagesTc], (ii / kStagesTc) & 1, status);
            }
        }
    } else if (warp == 1) {
        // ---------------- MMA issuer ----------------
        if (lane == 0) {
            int i = 0;
            for (long long t = blockIdx.x; t < ntiles; t += gridDim.x, ++i) {
                const int st = i % kStagesTc;
                const int acc = i % kEpiGroups;
                if (!mbar_wait(&full_bar[st], (i / kStagesTc) & 1, status)) break;
                if (!mbar_wait(&tempty_bar[acc], ((i / kEpiGroups) & 1) ^ 1, status)) break;
                tc_fence_after();
                const uint32_t a_base = smem_u32(ring + st * kTileBytes);
                const uint32_t b_base = smem_u32(hmat);
#pragma unroll
                for (int k = 0; k < kTile / 16; ++k) {
                    const uint32_t off = (k >> 2) * kHalfBytes + (k & 3) * 32;
                    mma_f16(tbase + acc * kTile, smem_desc_sw128(a_base + off),
                            smem_desc_sw128(b_base + off), kIdesc, k > 0);
                }
                mma_commit(&empty_bar[st]);
                mma_commit(&tfull_bar[acc]);
            }
        }
    } else {
        // ---------------- epilogue ----------------
        const int e = (warp - 2) >> 2;   // accumulator this group serves (tiles i = e mod 4)
        const int quad = warp & 3;       // TMEM lanes 32 quad .. 32 quad + 31
        const int m = quad * 32 + lane;  // group within the tile
        float mid[L - 1];
#pragma unroll
        for (int k = 0; k < L - 1; ++k) mid[k] = 0.5f * (__ldg(codebook + k) + __ldg(codebook + k + 1));
        BucketLookup bl{0u, 1.0f, false};
        if constexpr (B != 2) {
            bl = make_buckets<L>(mid, lane);
            if constexpr (!kChecked) bl.ok = true;
        }
        int i = e;
        JobCursor<NJ> cur;
        for (long long t = blockIdx.x + static_cast<long long>(e) * gridDim.x; t < ntiles;
             t += static_cast<long long>(kEpiGroups) * gridDim.x, i += kEpiGroups) {
            // warp-uniform decision: the TMEM loads below are .sync.aligned
            const bool ok = __all_sync(kFullMask, mbar_wait(&tfull_bar[e], (i / kEpiGroups) & 1, status));
            if (!ok) break;
            tc_fence_after();
            const uint32_t taddr = tbase + (static_cast<uint32_t>(quad * 32) << 16) + e * kTile;
            const int k = cur.at(jobs, t);
            const TcShape& sh = jobs.sh[k];
            const long long tl = t - jobs.tile0[k];
            const long long rb = tl % sh.tiles_r, j = tl / sh.tiles_r;
            const long long row = rb * kTile + m;
            const long long gid = row * sh.g_eff + j;
            // pass 1: the squared norm of the rotated group (32 TMEM columns at a time,
            // four independent partial sums)
            float ps[4] = {0.0f, 0.0f, 0.0f, 0.0f};
#pragma unroll
            for (int c = 0; c < kTile / 32; ++c) {
                float v[32];
                tmem_ld32(taddr + 32 * c, v);
                tmem_ld_wait();
#pragma unroll
                for (int q = 0; q < 32; ++q) ps[q & 3] = fmaf(v[q], v[q], ps[q & 3]);
            }
            const float ss = (ps[0] + ps[1]) + (ps[2] + ps[3]);
            const float nrm = sqrtf(ss);
            const float inv_n = nrm > 0.0f ? __frcp_rn(nrm) : 0.0f;  // u = r / n (0 for a zero group)
            float T[L - 1];
#pragma unroll
            for (int k = 0; k < L - 1; ++k) T[k] = nrm > 0.0f ? mid[k] * nrm : mid[k];
            // pass 2: indices, B words per 32 elements
            uint32_t words[4 * B];
#pragma unroll
            for (int c = 0; c < kTile / 32; ++c) {
                float v[32];
                tmem_ld32(taddr + 32 * c, v);
                tmem_ld_wait();
                if constexpr (B == 2) {
                    // ternary = the 2-bit form with a third threshold that nothing exceeds
                    float T3[3];
#pragma unroll
                    for (int k = 0; k < 3; ++k) T3[k] = k < L - 1 ? T[k < L - 1 ? k : 0] : __int_as_float(0x7f800000);
                    words[2 * c] = pack2_signbits<4, 0>(v, T3);
                    words[2 * c + 1] = pack2_signbits<4, 16>(v, T3);
                } else if constexpr (B == 3) {
#pragma unroll
                    for (int w = 0; w < B; ++w) words[B * c + w] = 0u;
                    if (bl.ok) {
#pragma unroll
                        for (int q = 0; q < 32; ++q) {
                            const uint32_t idx = bucket_index(v[q] * inv_n, bl);
                            const int bit = B * q, w = B * c + (bit >> 5), sh2 = bit & 31;
                            words[w] |= idx << sh2;
                            if (sh2 + B > 32) words[w + 1] |= idx >> (32 - sh2);
                        }
                    } else if constexpr (kChecked) {
#pragma unroll
                        for (int q = 0; q < 32; ++q) {
                            const uint32_t idx = nearest_index<L>(v[q], T);
                            const int bit = B * q, w = B * c + (bit >> 5), sh2 = bit & 31;
                            words[w] |= idx << sh2;
                            if (sh2 + B > 32) words[w + 1] |= idx >> (32 - sh2);
                        }
                    }
                } else {
                    // 32 / B fields per word, accumulated top-down: word = (word << B) + idx
                    if (bl.ok) {
#pragma unroll
                        for (int w = 0; w < B; ++w) {
                            uint32_t acc = 0u;
#pragma unroll
                            for (int q = 32 / B - 1; q >= 0; --q)
                                acc = (acc << B) + bucket_index(v[w * (32 / B) + q] * inv_n, bl);
                            words[B * c + w] = acc;
                        }
                    } else if constexpr (kChecked) {
#pragma unroll
                        for (int w = 0; w < B; ++w) {
                            uint32_t acc = 0u;
#pragma unroll
                            for (int q = 32 / B - 1; q >= 0; --q)
                                acc = (acc << B) + nearest_index<L>(v[w * (32 / B) + q], T);
                            words[B * c + w] = acc;
                        }
                    }
                }
            }
            tc_fence_before();
            __syncwarp();
            if (lane == 0) mbar_arrive(&tempty_bar[e]);
            if (row >= sh.r_eff) continue;
            uint4* dst = reinterpret_cast<uint4*>(jobs.packed[k] + gid * (16 * B));
#pragma unroll
            for (int p = 0; p < B; ++p)
                dst[p] = make_uint4(words[4 * p], words[4 * p + 1], words[4 * p + 2], words[4 * p + 3]);
            jobs.norms[k][gid] = __half_as_ushort(__float2half_rn(sqrtf(ss * 0.0078125f)));
        }
    }

    tc_fence_before();
    __syncthreads();
    if (warp == 1) {
        tc_fence_after();
        tmem_dealloc(tbase, kTmemCols);
    }
}

template <int B, int L, int NJ, bool kChecked>
cudaError_t launch_tc(const TcJobs<NJ>& jobs, const float* cb, unsigned* status, cudaStream_t st) {
    const int smem = (1 + kStagesTc) * kTileBytes + 1024;
    int dev = 0;
    cudaError_t e = cudaGetDevice(&dev);
    if (e != cudaSuccess) return e;
    static unsigned long long configured = 0;
    const unsigned long long bit = 1ull << (dev & 63);
    if (!(configured & bit)) {
        e = cudaFuncSetAttribute(quantize_tc_kernel<B, L, NJ, kChecked>, cudaFuncAttributeMaxDynamicSharedMemorySize, smem);
        if (e != cudaSuccess) return e;
        configured |= bit;
    }
    const long long ntiles = jobs.tile0[jobs.n];
    const int grid = static_cast<int>(std::max<long long>(1, std::min<long long>(ntiles, sm_count())));
    return launch_pdl(quantize_tc_kernel<B, L, NJ, kChecked>, dim3(grid), dim3(kTcThreads), smem, st, jobs, cb, status);
}

// Shape, tensor map and outputs of one tensor as job k of `jobs`.
template <int NJ>
bool add_job(TcJobs<NJ>& jobs, int k, const void* w, const Shape& sh, uint8_t* packed, uint16_t* norms) {
    const bool flat = sh.cols % kTile == 0;
    TcShape ts;
    ts.r_eff = flat ? sh.total_groups : sh.rows;
    const long long c_eff = flat ? kTile : sh.cols;
    ts.g_eff = flat ? 1 : sh.groups_per_row;
    ts.tiles_r = (ts.r_eff + kTile - 1) / kTile;
    ts.tiles = ts.tiles_r * ts.g_eff;
    const cuuint64_t gdim[2] = {static_cast<cuuint64_t>(c_eff), static_cast<cuuint64_t>(ts.r_eff)};
    const cuuint64_t gstride[1] = {static_cast<cuuint64_t>(c_eff) * 2};
    const cuuint32_t box[2] = {64, kTile};
    const cuuint32_t estride[2] = {1, 1};
    const CUresult r = tensor_map_encoder()(&jobs.map[k], CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, const_cast<void*>(w),
                                            gdim, gstride, box, estride, CU_TENSOR_MAP_INTERLEAVE_NONE,
                                            CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
                                            CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
    if (r != CUDA_SUCCESS) return false;
    jobs.sh[k] = ts;
    jobs.packed[k] = packed;
    jobs.norms[k] = norms;
    jobs.tile0[k + 1] = jobs.tile0[k] + ts.tiles;
    return true;
}

// The bucket table of make_buckets built on the host with the same fp32 operations: true when
// no bucket receives two midpoints of codebook c (L levels).
bool buckets_ok_host(const float* c, int L) {
    float mid[15];
    for (int k = 0; k < L - 1; ++k) mid[k] = 0.5f * (c[k] + c[k + 1]);
    float span = std::max(std::fabs(mid[0]), std::fabs(mid[L - 2])) * 1.1f;
    if (!(span > 0.0f)) span = 1.0f;
    const float sA = 0.5f / span;
    int cnt[32] = {0};
    for (int k = 0; k < L - 1; ++k) {
        float tt = std::fmaf(mid[k], sA, 0.5f);
        tt = tt > 0.0f ? (tt < 1.0f ? tt : 1.0f) : 0.0f;  // saturate (NaN -> 0)
        const float q = std::fmaf(tt, 31.0f, 12582912.0f);
        uint32_t bits = 0;
        std::memcpy(&bits, &q, sizeof(bits));
        if (++cnt[bits & 31u] > 1) return false;
    }
    return true;
}

// True when cb is this library's default codebook for `bits` and its bucket table is clean
// (then the kernel needs no in-kernel check and no select-tree fallback).
bool default_codebook_is_clean(int bits, const float* cb) {
    if (bits != 3 && bits != 4) return false;
    if (!is_default_codebook(bits, cb)) return false;
    static int clean[5] = {-1, -1, -1, -1, -1};  // per bits; the default codebooks never change
    static std::mutex mu;
    std::lock_guard<std::mutex> lock(mu);
    if (clean[bits] < 0) {
        float host[16] = {0};
        clean[bits] = (host_codebook(bits, kTile, 0, host) == (1 << bits) && buckets_ok_host(host, 1 << bits)) ? 1 : 0;
    }
    return clean[bits] == 1;
}

template <int NJ>
cudaError_t launch_bits(int bits, const TcJobs<NJ>& jobs, const float* cb, unsigned* status, cudaStream_t st) {
    const bool clean = default_codebook_is_clean(bits, cb);
    switch (bits) {
        case CQ_BITS_TERNARY: return launch_tc<2, 3, NJ, false>(jobs, cb, status, st);
        case 2: return launch_tc<2, 4, NJ, false>(jobs, cb, status, st);
        case 3:
            return clean ? launch_tc<3, 8, NJ, false>(jobs, cb, status, st) : launch_tc<3, 8, NJ, true>(jobs, cb, status, st);
        default:
            return clean ? launch_tc<4, 16, NJ, false>(jobs, cb, status, st) : launch_tc<4, 16, NJ, true>(jobs, cb, status, st);
    }
}

// Jobs per batched launch: the job list travels in the kernel parameters (at most 32 KB).
constexpr int kBatchJobs = 128;
static_assert(sizeof(TcJobs<kBatchJobs>) < 32000, "kernel parameter space");

}  // namespace

bool quantize_tc_supported(int w_dtype, const Shape& sh) {
    if (w_dtype != CQ_BF16 || sh.cols % 8 != 0) return false;
    const bool flat = sh.cols % kTile == 0;
    const long long r_eff = flat ? sh.total_groups : sh.rows;
    if (r_eff >= (1LL << 31)) return false;
    return tensor_map_encoder() != nullptr;
}

cudaError_t launch_quantize_tc(const void* w, const Shape& sh, int bits, const float* codebook,
                               uint8_t* packed, uint16_t* norms, unsigned* status,
                               cudaStream_t stream) {
    TcJobs<1> jobs;
    jobs.n = 1;
    jobs.tile0[0] = 0;
    if (!add_job(jobs, 0, w, sh, packed, norms)) return cudaErrorInvalidValue;
    return launch_bits(bits, jobs, codebook, status, stream);
}

cudaError_t launch_quantize_tc_batch(const QuantizeItem* items, int count, int bits,
                                     const float* codebook, unsigned* status, cudaStream_t stream) {
    static TcJobs<kBatchJobs> jobs;  // host staging (large); calls are serialised below
    static std::mutex mu;
    std::lock_guard<std::mutex> lock(mu);
    for (int i0 = 0; i0 < count; i0 += kBatchJobs) {
        const int n = std::min(kBatchJobs, count - i0);
        jobs.n = n;
        jobs.tile0[0] = 0;
        for (int k = 0; k < n; ++k) {
            const QuantizeItem& it = items[i0 + k];
            if (!add_job(jobs, k, it.w, it.sh, it.packed, it.norms)) return cudaErrorInvalidValue;
        }
        const cudaError_t e = launch_bits(bits, jobs, codebook, status, stream);
        if (e != cudaSuccess) return e;
    }
    return cudaSuccess;
}

}  // namespace cq
