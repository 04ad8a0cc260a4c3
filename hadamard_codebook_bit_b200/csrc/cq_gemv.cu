// cq_gemv.cu -- fused dequant-GEMV  y = W_hat x  without materialising W_hat.
//
// H is symmetric and orthonormal (pages "Cactus Quants CQ2-bit Quantization" and "How
// CQ2-bit Quantization Contributes to Needle 2's Small Footprint", "Hadamard Rotation"),
// so for group j of row r
//     <w_hat_rj, x_j> = <H (n_rj c[idx_rj]), x_j> = n_rj <c[idx_rj], H x_j>.
// Each activation group is rotated once; the packed weights are never expanded in memory.
//
// A job carries at most 8 activation rows (the MMA's N); larger batches, up to 64, arrive as
// one job per block of 8 rows with its own workspace slice (cq_api.cu).
//
// Step 1 (rotate_x_kernel, one block per group j, one warp per batch column b < 8):
//   x~_bj = H_int x_bj (zero for b >= batch), scaled by 2^-e_bj so its largest magnitude sits
//   in [2^13, 2^14), and written in the register-fragment order of the tensor-core B operand:
//   for 2-bit codes as a 16-bit integer X = 256 Xh + Xl in two int8 planes, for 3/4-bit codes
//   rounded to fp16.  The exponents go to an fp32 table.  Block 0 also writes the codeword
//   table (one exact power-of-two scale): int8 planes Ch, Cl of C = 256 Ch + Cl for 2-bit
//   codes, fp16 bytes for 3/4-bit codes.
//
// 2-bit codes (gemv_i8_kernel): m16n8k32 int8 MMAs with exact int32 accumulation per group;
// the A operand of a plane is one byte permute of a 4-entry table per four codes.  3/4-bit
// codes (gemv_split_kernel): m16n8k16 fp16 MMAs.  Both are launched as programmatic
// dependents of step 1 and share one structure: a block of S warps owns 16 output rows; warp
// w takes a contiguous chunk of about G / S groups, S chosen so that all row blocks are
// resident at once when they fit.  Per group a lane reads its 32 codes of rows g and g + 8
// straight from global memory (one coalesced 8/12/16-byte load per row, several groups in
// flight), builds the A fragments, runs the MMAs against x~, and folds the group's result
// into fp32 totals as  total += n_rj * 2^e_bj * acc.  The S warps' totals are summed in a
// fixed order, so the output is deterministic.
//
// K order inside a group.  The MMA contracts over the weights of a k-step in any order as
// long as A and B agree.  Lane (g, t) = (lane / 4, lane % 4) holds codes 32 t .. 32 t + 31 of
// each of its rows (bits 64 t .. 64 t + 63 of a 2-bit row block).
//   2-bit (int8, k-step of 32): in k-step s = 2 w + h, register r, byte q the lane takes
//             e = 32 t + 16 w + 8 h + 2 q + r: the codes that (word w >> (16 h + 2 r)) & 0x3333
//             places in selector nibbles q = 0..3.
//   3/4-bit (fp16, k-step of 16): four weights q = 0..3 (MMA k = 2t, 2t+1, 2t+8, 2t+9) are
//             e = 32 t + 4 s + q: four adjacent codes, one 12- or 16-bit field spread to nibble
//             selectors and looked up with byte permutes in 8 / 16-entry byte tables.
#include <algorithm>
#include <mutex>

#include "cq_device.cuh"
#include "cq_internal.h"

namespace cq {
namespace {

using namespace dev;

constexpr int kRotThreads = 256;  // 8 warps = 8 batch columns
constexpr int kRowsPerBlock = 16;
constexpr int kBatchCols = 8;     // MMA N: batch columns, zero padded
constexpr int kXEntry = 8;        // bytes of B fragment per lane per k-step (4 fp16)

// Workspace: [G][4 k-step pairs][32 lanes] of 8 fp16 | fp32 exponents [G][8] | codeword table.
__host__ __device__ inline size_t frag_bytes(long long G) { return static_cast<size_t>(G) * 8 * 32 * kXEntry; }
__host__ __device__ inline size_t scale_bytes(long long G) { return static_cast<size_t>(G) * kBatchCols * sizeof(float); }

struct CodeTable {
    uint32_t lo, hi;      // codes 0..3: int8 bytes of Ch / Cl (2-bit codes), else low / high fp16 bytes
    float inv_scale;      // 2^-cs: the table holds fp16(c_k 2^cs)
    uint32_t pad;
    uint16_t h[16];       // fp16 codewords 0..15 (entries past L repeat the last level)
};

__device__ __forceinline__ uint32_t prmt(uint32_t a, uint32_t b, uint32_t sel) {
    uint32_t d;
    asm("prmt.b32 %0, %1, %2, %3;" : "=r"(d) : "r"(a), "r"(b), "r"(sel));
    return d;
}


__device__ __forceinline__ uint32_t pack_half2(float lo, float hi) {
    return static_cast<uint32_t>(__half_as_ushort(__float2half_rn(lo))) |
           (static_cast<uint32_t>(__half_as_ushort(__float2half_rn(hi))) << 16);
}

__device__ __forceinline__ void mma_16816(float (&c)[4], uint32_t a0, uint32_t a1, uint32_t a2,
                                          uint32_t a3, uint32_t b0, uint32_t b1) {
    asm volatile(
        "mma.sync.aligned.m16n8k16.row.col.f32.f16.f16.f32 {%0, %1, %2, %3}, {%4, %5, %6, %7}, "
        "{%8, %9}, {%0, %1, %2, %3};"
        : "+f"(c[0]), "+f"(c[1]), "+f"(c[2]), "+f"(c[3])
        : "r"(a0), "r"(a1), "r"(a2), "r"(a3), "r"(b0), "r"(b1));
}

// The products of one launch (one for cq_dequant_gemv, up to kGemvBatch for the batched
// call).  Job k owns rotation blocks [group0[k], group0[k + 1]) (one per group) and GEMV blocks
// [block0[k], block0[k + 1]) (one per 16 rows); its workspace holds x~ fragments, exponents and
// the codeword table in that order.
template <int NJ>
struct GemvJobs {
    const uint16_t* x[NJ];
    const uint8_t* packed[NJ];
    const uint16_t* norms[NJ];
    char* ws[NJ];
    float* y[NJ];
    long long rows[NJ];
    long long cols[NJ];
    int G[NJ];
    int batch[NJ];
    long long group0[NJ + 1];
    long long block0[NJ + 1];
    int n;
};

// Largest k < n with prefix[k] <= v (v < prefix[n]).
template <int NJ>
__device__ __forceinline__ int find_job(const long long (&prefix)[NJ + 1], int n, long long v) {
    if constexpr (NJ == 1) {
        return 0;
    } else {
        int lo = 0, hi = n - 1;
        while (lo < hi) {
            const int mid = (lo + hi + 1) >> 1;
            if (prefix[mid] <= v) lo = mid;
            else hi = mid - 1;
        }
        return lo;
    }
}

// ---------------------------------------------------------------------------------------
// step 1: rotate the activations into fragment order (+ codeword table)
// ---------------------------------------------------------------------------------------

template <int B, int L, int NJ>
__global__ void __launch_bounds__(kRotThreads)
    rotate_x_kernel(const __grid_constant__ GemvJobs<NJ> jobs, const float* __restrict__ codebook) {
    pdl_trigger();  // the GEMV may be scheduled now; it waits for this kernel before any access
    pdl_wait();
    const int jk = find_job<NJ>(jobs.group0, jobs.n, blockIdx.x);
    const long long j = blockIdx.x - jobs.group0[jk];
    const uint16_t* __restrict__ x = jobs.x[jk];
    const long long cols = jobs.cols[jk], G = jobs.G[jk];
    const int batch = jobs.batch[jk];
    __half* __restrict__ xfrag = reinterpret_cast<__half*>(jobs.ws[jk]);
    float* __restrict__ xscale = reinterpret_cast<float*>(jobs.ws[jk] + frag_bytes(G));
    CodeTable* __restrict__ table = reinterpret_cast<CodeTable*>(jobs.ws[jk] + frag_bytes(G) + scale_bytes(G));
    const int b = threadIdx.x >> 5, lane = threadIdx.x & 31;

    if (j == 0 && threadIdx.x < 32) {
        float m = 0.0f;
#pragma unroll
        for (int k = 0; k < L; ++k) m = fmaxf(m, fabsf(__ldg(codebook + k)));
        const int cs = (m > 0.0f) ? (13 - ilogbf(m)) : 0;
        const int k = threadIdx.x < 16 ? (threadIdx.x < L ? static_cast<int>(threadIdx.x) : L - 1) : 0;
        const uint32_t u = __half_as_ushort(__float2half_rn(ldexpf(__ldg(codebook + k), cs)));
        if (threadIdx.x < 16) table->h[threadIdx.x] = static_cast<uint16_t>(u);
        uint32_t lo = 0, hi = 0;
        if constexpr (B == 2) {
            // 2-bit codes: integer codewords C = rint(c 2^cs) (|C| < 2^14) split as
            // C = 256 Ch + Cl, Ch in [-64, 64], Cl in [-128, 127]; lo / hi hold the int8
            // bytes of Ch / Cl for codes 0..3
            const int cq = __float2int_rn(ldexpf(__ldg(codebook + (threadIdx.x < 4 ? k : 0)), cs));
            const int ch = (cq + 128) >> 8, cl = cq - (ch << 8);
#pragma unroll
            for (int q = 0; q < 4; ++q) {
                const uint32_t hq = static_cast<uint32_t>(__shfl_sync(kFullMask, ch, q)) & 0xffu;
                const uint32_t lq = static_cast<uint32_t>(__shfl_sync(kFullMask, cl, q)) & 0xffu;
                lo |= hq << (8 * q);
                hi |= lq << (8 * q);
            }
        } else {
            // bytes of the fp16 codewords 0..3 gathered in every lane
#pragma unroll
            for (int q = 0; q < 4; ++q) {
                const uint32_t uq = __shfl_sync(kFullMask, u, q);
                lo |= (uq & 0xffu) << (8 * q);
                hi |= (uq >> 8) << (8 * q);
            }
        }
        if (threadIdx.x == 0) {
            table->lo = lo;
            table->hi = hi;
            table->inv_scale = ldexpf(1.0f, -cs);
            table->pad = 0;
        }
    }

    // lane l holds elements 4l..4l+3 of column b of group j
    float v[4] = {0.0f, 0.0f, 0.0f, 0.0f};
    if (b < batch) {
        const long long c0 = j * 128 + 4 * lane;
        const uint16_t* src = x + static_cast<long long>(b) * cols + c0;
#pragma unroll
        for (int i = 0; i < 4; ++i)
            if (c0 + i < cols) v[i] = bf16_bits_to_float(__ldg(src + i));
    }
    {  // element bits 0-1 in registers
        const float a0 = v[0] + v[1], a1 = v[0] - v[1], a2 = v[2] + v[3], a3 = v[2] - v[3];
        v[0] = a0 + a2;
        v[1] = a1 + a3;
        v[2] = a0 - a2;
        v[3] = a1 - a3;
    }
#pragma unroll
    for (int m = 1; m < 32; m <<= 1) {  // element bits 2-6 across lanes
        const float sg = (lane & m) ? -1.0f : 1.0f;
#pragma unroll
        for (int i = 0; i < 4; ++i) v[i] = fmaf(v[i], sg, __shfl_xor_sync(kFullMask, v[i], m));
    }
    float mx = fmaxf(fmaxf(fabsf(v[0]), fabsf(v[1])), fmaxf(fabsf(v[2]), fabsf(v[3])));
#pragma unroll
    for (int m = 16; m >= 1; m >>= 1) mx = fmaxf(mx, __shfl_xor_sync(kFullMask, mx, m));
    const int e = (mx > 0.0f) ? (ilogbf(mx) - 13) : 0;
    const float down = ldexpf(1.0f, -e);
    if (lane == 0) xscale[j * kBatchCols + b] = ldexpf(1.0f, e);
    // element e = 4 lane + i  ->  (k-step s, lane 4 b + t, half q); entry layout
    // [j][s / 2][lane][8 halves], halves 4 (s % 2) + q
    const int t = lane >> 3;
    if constexpr (B == 2) {
        // 16-bit integer X = rint(x~ 2^-e) = 256 Xh + Xl as two int8 planes, planes h / l of
        // batch column b being B columns 2 (b % 4), 2 (b % 4) + 1 of n-tile b / 4.  Element e
        // of the group goes to lane t = e / 32 of k-step s = 2 ((e / 16) % 2) + (e / 8) % 2,
        // register r = e % 2, byte (e / 2) % 4 (the order in which the GEMV decodes the codes).
        // Entry layout: [group][n-tile][lane][k-step][r][byte], 32 bytes per lane.
        uint8_t* xb = reinterpret_cast<uint8_t*>(xfrag);
        const int nt = b >> 2, nl = 2 * (b & 3);
#pragma unroll
        for (int i = 0; i < 4; ++i) {
            const int e = 4 * lane + i;
            const int xq = __float2int_rn(v[i] * down);
            const int xh = (xq + 128) >> 8, xl = xq - (xh << 8);
            const int t = e >> 5, ks = 2 * ((e >> 4) & 1) + ((e >> 3) & 1), r = e & 1, by = (e >> 1) & 3;
            const long long o = ((j * 2 + nt) * 32 + 4 * nl + t) * 32 + ks * 8 + 4 * r + by;
            xb[o] = static_cast<uint8_t>(xh);
            xb[o + 4 * 32] = static_cast<uint8_t>(xl);  // lane + 4: B column nl + 1
        }
    } else {
        const int s = lane & 7;
        const uint32_t h01 = pack_half2(v[0] * down, v[1] * down), h23 = pack_half2(v[2] * down, v[3] * down);
        *reinterpret_cast<uint2*>(xfrag + ((j * 4 + (s >> 1)) * 32 + 4 * b + t) * 8 + 4 * (s & 1)) =
            make_uint2(h01, h23);
    }
}

// ---------------------------------------------------------------------------------------
// step 2: streaming tensor-core GEMV
// ---------------------------------------------------------------------------------------

// Codes of one lane for one group row: words 2t, 2t+1 (2-bit), 3t..3t+2 (3-bit), 4t..4t+3.
template <int B>
struct Seg {
    uint32_t w[B];
};

template <int B>
__device__ __forceinline__ Seg<B> load_seg(const uint8_t* __restrict__ blk, int t, bool ok) {
    Seg<B> r;
    if (!ok) {
#pragma unroll
        for (int i = 0; i < B; ++i) r.w[i] = 0u;
        return r;
    }
    if constexpr (B == 2) {
        asm volatile("ld.global.nc.L1::no_allocate.v2.u32 {%0, %1}, [%2];"
                     : "=r"(r.w[0]), "=r"(r.w[1])
                     : "l"(blk + 8 * t));
    } else if constexpr (B == 4) {
        const uint4 v = ld_stream16(blk + 16 * t);
        r.w[0] = v.x;
        r.w[1] = v.y;
        r.w[2] = v.z;
        r.w[3] = v.w;
    } else {
#pragma unroll
        for (int i = 0; i < 3; ++i)
            asm volatile("ld.global.nc.L1::no_allocate.u32 %0, [%1];" : "=r"(r.w[i]) : "l"(blk + 12 * t + 4 * i));
    }
    return r;
}

// Byte tables of the fp16 codewords (3/4-bit codes): lo[k] / hi[k] hold the low / high
// bytes of codes 4k..4k+3.
struct ByteTables {
    uint32_t lo[4], hi[4];
};

// A-fragment registers of one row in k-step S: r0 = (c[k=2t], c[2t+1]), r1 = (c[2t+8], c[2t+9]).
template <int B, int S>
__device__ __forceinline__ void decode(const Seg<B>& sg, const ByteTables& tb, uint32_t& r0, uint32_t& r1) {
    static_assert(B == 3 || B == 4, "2-bit codes take the int8 path");
    {
        uint32_t sel, m = 0x3210u;
        uint32_t lo4, hi4;
        if constexpr (B == 4) {
            const uint32_t f = (S & 1) ? (sg.w[S >> 1] >> 16) : sg.w[S >> 1];  // 4 codes in nibbles
            sel = f & 0x7777u;
            m |= (f >> 1) & 0x4444u;  // code >= 8: take the byte from the upper 8-entry half
            lo4 = prmt(prmt(tb.lo[0], tb.lo[1], sel), prmt(tb.lo[2], tb.lo[3], sel), m);
            hi4 = prmt(prmt(tb.hi[0], tb.hi[1], sel), prmt(tb.hi[2], tb.hi[3], sel), m);
        } else {
            constexpr int kBit = 12 * S;  // four 3-bit codes at bits 12 S .. 12 S + 11
            uint32_t f;
            if constexpr ((kBit & 31) + 12 <= 32) {
                f = sg.w[kBit >> 5] >> (kBit & 31);
            } else {
                f = __funnelshift_r(sg.w[kBit >> 5], sg.w[(kBit >> 5) + 1], kBit & 31);
            }
            sel = (f & 0x7u) | ((f << 1) & 0x70u) | ((f << 2) & 0x700u) | ((f << 3) & 0x7000u);
            lo4 = prmt(tb.lo[0], tb.lo[1], sel);
            hi4 = prmt(tb.hi[0], tb.hi[1], sel);
        }
        r0 = prmt(lo4, hi4, 0x5140u);
        r1 = prmt(lo4, hi4, 0x7362u);
    }
}

__device__ __forceinline__ uint4 ld_v4_volatile(const void* p) {
    uint4 r;
    asm volatile("ld.global.v4.u32 {%0, %1, %2, %3}, [%4];"
                 : "=r"(r.x), "=r"(r.y), "=r"(r.z), "=r"(r.w)
                 : "l"(p));
    return r;
}

// Byte tables and scale from the codeword table step 1 wrote (volatile loads: see load_bfrag).
template <int B>
__device__ __forceinline__ void load_tables(const CodeTable* table, ByteTables& tb, float& inv_scale) {
    const uint4 head = ld_v4_volatile(table);  // lo, hi, inv_scale, pad
    inv_scale = __uint_as_float(head.z);
    {
        const uint4 h0 = ld_v4_volatile(reinterpret_cast<const uint8_t*>(table) + 16);  // h[0..7]
        const uint4 h1 = ld_v4_volatile(reinterpret_cast<const uint8_t*>(table) + 32);  // h[8..15]
        const uint32_t hw[8] = {h0.x, h0.y, h0.z, h0.w, h1.x, h1.y, h1.z, h1.w};
#pragma unroll
        for (int k = 0; k < 4; ++k) {
            // codes 4k..4k+3 = words 2k, 2k+1 (two fp16 each)
            const uint32_t a = hw[2 * k], c = hw[2 * k + 1];
            tb.lo[k] = prmt(a, c, 0x6420u);  // low bytes
            tb.hi[k] = prmt(a, c, 0x7531u);  // high bytes
        }
    }
}

constexpr int kMaxSplit = 16;  // warps per block
// groups per warp in flight (fewer for the wider 3/4-bit code words)
template <int B>
constexpr int kDepth = B == 2 ? 8 : 4;

// B fragments of one group (four k-step pairs); lanes holding padding columns skip the loads
// and keep the zeros they were initialised with.  Everything step 1 writes is read with
// volatile asm so that no read can be moved above the griddepcontrol.wait.
__device__ __forceinline__ void load_bfrag(const uint4* __restrict__ p, bool on, uint4 (&bf)[4]) {
#pragma unroll
    for (int sp = 0; sp < 4; ++sp)
        asm volatile(
            "{\n\t.reg .pred q;\n\t"
            "setp.ne.u32 q, %4, 0;\n\t"
            "@q ld.global.nc.v4.u32 {%0, %1, %2, %3}, [%5];\n\t}"
            : "+r"(bf[sp].x), "+r"(bf[sp].y), "+r"(bf[sp].z), "+r"(bf[sp].w)
            : "r"(static_cast<uint32_t>(on)), "l"(p + sp * 32));
}

// One warp's walk over its chunk of groups for 16 rows (rows past the end read row 0 and are
// dropped at the end, so no load is predicated on the row).
template <int B>
struct GemvWarp {
    static constexpr int kBlk = 16 * B;
    const uint8_t* pa;   // packed block of row g at the current group
    const uint8_t* pb;   // ... row g + 8
    const uint16_t* na;  // norms of row g at the current group
    const uint16_t* nb;
    const uint4* xf;     // B fragments of the current group, this lane
    const float2* xs;    // exponents of the current group, columns 2t, 2t + 1
    bool bcol;           // this lane holds a real batch column
    int t;
    ByteTables tb;
    uint4 bf[4];
    float tot[4];

    // kDepth<B> groups (or the first n of them when !kFull): all loads first, then the math
    template <bool kFull>
    __device__ __forceinline__ void batch(int n) {
        Seg<B> ca[kDepth<B>], cb[kDepth<B>];
        float sa[kDepth<B>], sb[kDepth<B>];
#pragma unroll
        for (int u = 0; u < kDepth<B>; ++u) {
            const bool on = kFull || u < n;
            ca[u] = load_seg<B>(pa + u * kBlk, t, on);
            cb[u] = load_seg<B>(pb + u * kBlk, t, on);
            sa[u] = on ? __half2float(__ushort_as_half(__ldg(na + u))) : 0.0f;
            sb[u] = on ? __half2float(__ushort_as_half(__ldg(nb + u))) : 0.0f;
        }
#pragma unroll
        for (int u = 0; u < kDepth<B>; ++u) {
            if (!kFull && u >= n) break;
            load_bfrag(xf + u * 128, bcol, bf);
            float2 x2;  // volatile: stays after the dependency wait
            asm volatile("ld.global.nc.v2.f32 {%0, %1}, [%2];" : "=f"(x2.x), "=f"(x2.y) : "l"(xs + u * 4));
            float acc[4] = {0.0f, 0.0f, 0.0f, 0.0f};
            uint32_t a0, a1, a2, a3;
#define CQ_KSTEP(SS, B0, B1)                   \
    decode<B, SS>(ca[u], tb, a0, a2);          \
    decode<B, SS>(cb[u], tb, a1, a3);          \
    mma_16816(acc, a0, a1, a2, a3, B0, B1);
            CQ_KSTEP(0, bf[0].x, bf[0].y)
            CQ_KSTEP(1, bf[0].z, bf[0].w)
            CQ_KSTEP(2, bf[1].x, bf[1].y)
            CQ_KSTEP(3, bf[1].z, bf[1].w)
            CQ_KSTEP(4, bf[2].x, bf[2].y)
            CQ_KSTEP(5, bf[2].z, bf[2].w)
            CQ_KSTEP(6, bf[3].x, bf[3].y)
            CQ_KSTEP(7, bf[3].z, bf[3].w)
#undef CQ_KSTEP
            tot[0] = fmaf(sa[u] * x2.x, acc[0], tot[0]);
            tot[1] = fmaf(sa[u] * x2.y, acc[1], tot[1]);
            tot[2] = fmaf(sb[u] * x2.x, acc[2], tot[2]);
            tot[3] = fmaf(sb[u] * x2.y, acc[3], tot[3]);
        }
        pa += kDepth<B> * kBlk;
        pb += kDepth<B> * kBlk;
        na += kDepth<B>;
        nb += kDepth<B>;
        xf += kDepth<B> * 128;
        xs += kDepth<B> * 4;
    }
};

__device__ __forceinline__ void mma_i8(int (&c)[4], uint32_t a0, uint32_t a1, uint32_t a2, uint32_t a3,
                                       uint32_t b0, uint32_t b1) {
    asm volatile(
        "mma.sync.aligned.m16n8k32.row.col.s32.s8.s8.s32 {%0, %1, %2, %3}, {%4, %5, %6, %7}, "
        "{%8, %9}, {%0, %1, %2, %3};"
        : "+r"(c[0]), "+r"(c[1]), "+r"(c[2]), "+r"(c[3])
        : "r"(a0), "r"(a1), "r"(a2), "r"(a3), "r"(b0), "r"(b1));
}

// 2-bit codes on the int8 tensor cores.  C = 256 Ch + Cl (codewords) and X = 256 Xh + Xl
// (rotated activations) are 16-bit integers in two int8 planes each; for a k-step the A
// operand of plane P is one byte permute of the 4-entry table of P per four codes, with the
// codes as nibble selectors straight from the packed word (w >> (16 hi + 2 r)) & 0x3333.  B
// holds Xh and Xl of batch column b in columns 2 (b % 4) and 2 (b % 4) + 1, so lane t's
// accumulators are the four cross products of batch column t (+ 4 per extra n-tile), combined
// per group in fp32 as 65536 ChXh + 256 (ChXl + ClXh) + ClXl.
template <int NT>
struct GemvWarpI8 {
    static constexpr int kBlk = 32;
    static constexpr int kD = 4;  // groups of codes in flight per warp
    const uint8_t* pa;
    const uint8_t* pb;
    const uint16_t* na;
    const uint16_t* nb;
    const uint4* xf;   // this lane's 32 bytes of B fragments of n-tile 0 of the current group
    const float* xs;   // exponents 2^e of the current group (8 columns)
    bool bcol[NT];     // lane holds a real B column in n-tile nt
    int t;
    uint32_t th, tl;   // int8 bytes of Ch / Cl for codes 0..3
    float tot[NT][2];  // batch column t + 4 nt, rows g and g + 8

    template <bool kFull>
    __device__ __forceinline__ void batch(int n) {
        Seg<2> ca[kD], cb[kD];
        float sa[kD], sb[kD];
#pragma unroll
        for (int u = 0; u < kD; ++u) {
            const bool on = kFull || u < n;
            ca[u] = load_seg<2>(pa + u * kBlk, t, on);
            cb[u] = load_seg<2>(pb + u * kBlk, t, on);
            sa[u] = on ? __half2float(__ushort_as_half(__ldg(na + u))) : 0.0f;
            sb[u] = on ? __half2float(__ushort_as_half(__ldg(nb + u))) : 0.0f;
        }
#pragma unroll
        for (int u = 0; u < kD; ++u) {
            if (!kFull && u >= n) break;
            uint4 bq[NT][2];
#pragma unroll
            for (int nt = 0; nt < NT; ++nt) {
                bq[nt][0] = bq[nt][1] = make_uint4(0, 0, 0, 0);
                const uint4* p = xf + u * 128 + nt * 64;
                asm volatile(
                    "{\n\t.reg .pred q;\n\t"
                    "setp.ne.u32 q, %8, 0;\n\t"
                    "@q ld.global.nc.v4.u32 {%0, %1, %2, %3}, [%9];\n\t"
                    "@q ld.global.nc.v4.u32 {%4, %5, %6, %7}, [%10];\n\t}"
                    : "+r"(bq[nt][0].x), "+r"(bq[nt][0].y), "+r"(bq[nt][0].z), "+r"(bq[nt][0].w),
                      "+r"(bq[nt][1].x), "+r"(bq[nt][1].y), "+r"(bq[nt][1].z), "+r"(bq[nt][1].w)
                    : "r"(static_cast<uint32_t>(bcol[nt])), "l"(p), "l"(p + 1));
            }
            float xsv[NT];
#pragma unroll
            for (int nt = 0; nt < NT; ++nt)
                asm volatile("ld.global.nc.f32 %0, [%1];" : "=f"(xsv[nt]) : "l"(xs + u * 8 + t + 4 * nt));
            int ah[NT][4], al[NT][4];
#pragma unroll
            for (int nt = 0; nt < NT; ++nt)
#pragma unroll
                for (int q = 0; q < 4; ++q) ah[nt][q] = al[nt][q] = 0;
#pragma unroll
            for (int ks = 0; ks < 4; ++ks) {
                const int wsel = ks >> 1, sh = 16 * (ks & 1);
                const uint32_t sa0 = (ca[u].w[wsel] >> sh) & 0x3333u, sa1 = (ca[u].w[wsel] >> (sh + 2)) & 0x3333u;
                const uint32_t sb0 = (cb[u].w[wsel] >> sh) & 0x3333u, sb1 = (cb[u].w[wsel] >> (sh + 2)) & 0x3333u;
                const uint32_t h0 = prmt(th, th, sa0), h1 = prmt(th, th, sb0), h2 = prmt(th, th, sa1), h3 = prmt(th, th, sb1);
                const uint32_t l0 = prmt(tl, tl, sa0), l1 = prmt(tl, tl, sb0), l2 = prmt(tl, tl, sa1), l3 = prmt(tl, tl, sb1);
#pragma unroll
                for (int nt = 0; nt < NT; ++nt) {
                    const uint4& q = bq[nt][ks >> 1];
                    const uint32_t b0 = (ks & 1) ? q.z : q.x, b1 = (ks & 1) ? q.w : q.y;
                    mma_i8(ah[nt], h0, h1, h2, h3, b0, b1);
                    mma_i8(al[nt], l0, l1, l2, l3, b0, b1);
                }
            }
#pragma unroll
            for (int nt = 0; nt < NT; ++nt) {
                const float va = fmaf(static_cast<float>(ah[nt][0]), 65536.0f,
                                      fmaf(static_cast<float>(ah[nt][1] + al[nt][0]), 256.0f, static_cast<float>(al[nt][1])));
                const float vb = fmaf(static_cast<float>(ah[nt][2]), 65536.0f,
                                      fmaf(static_cast<float>(ah[nt][3] + al[nt][2]), 256.0f, static_cast<float>(al[nt][3])));
                tot[nt][0] = fmaf(sa[u] * xsv[nt], va, tot[nt][0]);
                tot[nt][1] = fmaf(sb[u] * xsv[nt], vb, tot[nt][1]);
            }
        }
        pa += kD * kBlk;
        pb += kD * kBlk;
        na += kD;
        nb += kD;
        xf += kD * 128;
        xs += kD * 8;
    }
};

template <int B, int NJ>
__global__ void __maxnreg__(96)
    gemv_split_kernel(const __grid_constant__ GemvJobs<NJ> jobs) {
    __shared__ float4 red[kMaxSplit][32];
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int S = static_cast<int>(blockDim.x >> 5);
    const int g = lane >> 2, t = lane & 3;
    const int jk = find_job<NJ>(jobs.block0, jobs.n, blockIdx.x);
    const uint8_t* __restrict__ packed = jobs.packed[jk];
    const uint16_t* __restrict__ norms = jobs.norms[jk];
    const long long rows = jobs.rows[jk];
    const int G = jobs.G[jk], batch = jobs.batch[jk];
    float* __restrict__ y = jobs.y[jk];
    const uint4* xfrag = reinterpret_cast<const uint4*>(jobs.ws[jk]);
    const float2* xscale = reinterpret_cast<const float2*>(jobs.ws[jk] + frag_bytes(G));
    const CodeTable* table = reinterpret_cast<const CodeTable*>(jobs.ws[jk] + frag_bytes(G) + scale_bytes(G));
    const long long r0 = (blockIdx.x - jobs.block0[jk]) * kRowsPerBlock;
    const long long ra = r0 + g, rb = r0 + g + 8;
    const bool oka = ra < rows, okb = rb < rows;

    // this warp's groups: [jb, je)
    const int chunk = (G + S - 1) / S;
    const int jb = min(G, warp * chunk), je = min(G, jb + chunk);

    GemvWarp<B> st;
    st.pa = packed + ((oka ? ra : 0) * G + jb) * GemvWarp<B>::kBlk;
    st.pb = packed + ((okb ? rb : 0) * G + jb) * GemvWarp<B>::kBlk;
    st.na = norms + (oka ? ra : 0) * G + jb;
    st.nb = norms + (okb ? rb : 0) * G + jb;
    st.xf = xfrag + static_cast<long long>(jb) * 128 + lane;
    st.xs = xscale + static_cast<long long>(jb) * 4 + t;
    st.bcol = g < batch;
    st.t = t;
#pragma unroll
    for (int sp = 0; sp < 4; ++sp) st.bf[sp] = make_uint4(0, 0, 0, 0);
    st.tot[0] = st.tot[1] = st.tot[2] = st.tot[3] = 0.0f;

    // Nothing is read before the dependency wait: loads issued earlier by a programmatic
    // dependent (even of buffers written by kernels that ran before step 1) returned stale
    // data on this hardware.  The early launch still hides the launch latency.  (An L2
    // prefetch of the codes here measured ~1 us slower per call.)
    pdl_trigger();
    pdl_wait();
    float inv_scale;
    load_tables<B>(table, st.tb, inv_scale);

    int n = je - jb;
    for (; n >= kDepth<B>; n -= kDepth<B>) st.template batch<true>(n);
    if (n > 0) st.template batch<false>(n);

    float4 a = make_float4(st.tot[0], st.tot[1], st.tot[2], st.tot[3]);
    if (S > 1) {
        red[warp][lane] = a;
        __syncthreads();
        if (warp != 0) return;
        a = red[0][lane];
        for (int w = 1; w < S; ++w) {
            const float4 b = red[w][lane];
            a.x += b.x;
            a.y += b.y;
            a.z += b.z;
            a.w += b.w;
        }
    }
    const float f = inv_scale * kInvSqrt128;
    const int c0 = 2 * t, c1 = 2 * t + 1;
    if (oka && c0 < batch) y[c0 * rows + ra] = a.x * f;
    if (oka && c1 < batch) y[c1 * rows + ra] = a.y * f;
    if (okb && c0 < batch) y[c0 * rows + rb] = a.z * f;
    if (okb && c1 < batch) y[c1 * rows + rb] = a.w * f;
}

// 2-bit codes: the same block / split structure as gemv_split_kernel on the int8 path.
// Four groups of codes in flight and a 72-register cap (batch <= 4) give up to 28 resident
// warps per SM; the split-K buffer is dynamic (512 bytes per warp of the block) so that the
// common one-warp blocks leave the shared-memory carve-out, and with it the L1 space that
// holds the rotated activations, nearly whole.  (Measured on a 112-product 7B-scale mix:
// 0.312 -> 0.291 ms against 8 groups, 96 registers and a static 8 KB buffer.)
template <int NT, int NJ>
__global__ void __maxnreg__(NT == 1 ? 72 : 96)
    gemv_i8_kernel(const __grid_constant__ GemvJobs<NJ> jobs) {
    extern __shared__ float4 red_i8[];  // [S][32], S = warps of the block
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int S = static_cast<int>(blockDim.x >> 5);
    const int g = lane >> 2, t = lane & 3;
    const int jk = find_job<NJ>(jobs.block0, jobs.n, blockIdx.x);
    const uint8_t* __restrict__ packed = jobs.packed[jk];
    const uint16_t* __restrict__ norms = jobs.norms[jk];
    const long long rows = jobs.rows[jk];
    const int G = jobs.G[jk], batch = jobs.batch[jk];
    float* __restrict__ y = jobs.y[jk];
    const uint4* xfrag = reinterpret_cast<const uint4*>(jobs.ws[jk]);
    const float* xscale = reinterpret_cast<const float*>(jobs.ws[jk] + frag_bytes(G));
    const CodeTable* table = reinterpret_cast<const CodeTable*>(jobs.ws[jk] + frag_bytes(G) + scale_bytes(G));
    const long long r0 = (blockIdx.x - jobs.block0[jk]) * kRowsPerBlock;
    const long long ra = r0 + g, rb = r0 + g + 8;
    const bool oka = ra < rows, okb = rb < rows;
    const int chunk = (G + S - 1) / S;
    const int jb = min(G, warp * chunk), je = min(G, jb + chunk);

    GemvWarpI8<NT> st;
    st.pa = packed + ((oka ? ra : 0) * G + jb) * 32;
    st.pb = packed + ((okb ? rb : 0) * G + jb) * 32;
    st.na = norms + (oka ? ra : 0) * G + jb;
    st.nb = norms + (okb ? rb : 0) * G + jb;
    st.xf = xfrag + static_cast<long long>(jb) * 128 + 2 * lane;
    st.xs = xscale + static_cast<long long>(jb) * 8;
#pragma unroll
    for (int nt = 0; nt < NT; ++nt) {
        st.bcol[nt] = (g >> 1) + 4 * nt < batch;
        st.tot[nt][0] = st.tot[nt][1] = 0.0f;
    }
    st.t = t;

    // no global access before the dependency wait (see gemv_split_kernel)
    pdl_trigger();
    pdl_wait();
    const uint4 head = ld_v4_volatile(table);  // Ch bytes, Cl bytes, 2^-cs, pad
    st.th = head.x;
    st.tl = head.y;
    const float inv_scale = __uint_as_float(head.z);

    int n = je - jb;
    constexpr int kD = GemvWarpI8<NT>::kD;
    for (; n >= kD; n -= kD) st.template batch<true>(n);
    if (n > 0) st.template batch<false>(n);

    float4 a = make_float4(st.tot[0][0], st.tot[0][1], NT > 1 ? st.tot[NT - 1][0] : 0.0f,
                           NT > 1 ? st.tot[NT - 1][1] : 0.0f);
    if (S > 1) {
        red_i8[warp * 32 + lane] = a;
        __syncthreads();
        if (warp != 0) return;
        a = red_i8[lane];
        for (int w = 1; w < S; ++w) {
            const float4 b = red_i8[w * 32 + lane];
            a.x += b.x;
            a.y += b.y;
            a.z += b.z;
            a.w += b.w;
        }
    }
    const float f = inv_scale * kInvSqrt128;
    // lane (g, t) holds rows g and g + 8 of batch column t (and t + 4)
    if (t < batch) {
        if (oka) y[t * rows + ra] = a.x * f;
        if (okb) y[t * rows + rb] = a.y * f;
    }
    if (NT > 1 && t + 4 < batch) {
        if (oka) y[(t + 4) * rows + ra] = a.z * f;
        if (okb) y[(t + 4) * rows + rb] = a.w * f;
    }
}

// Registers per thread of gemv_split_kernel<B, NJ> on the current device (queried once).
template <int B, int NJ>
int gemv_regs() {
    static int regs = 0;
    if (regs == 0) {
        cudaFuncAttributes fa;
        regs = (cudaFuncGetAttributes(&fa, gemv_split_kernel<B, NJ>) == cudaSuccess && fa.numRegs > 0) ? fa.numRegs : 128;
    }
    return regs;
}

// Warps per block.  The row blocks are spread over the SMs in one round when they fit:
// every SM holds ceil(blocks / SMs) of them, and the split is the largest (up to 16 warps,
// at least two groups a warp of the narrowest job) for which that many blocks stay resident
// by registers.
int gemv_split(long long blocks, long long G, int regs) {
    const long long sms = sm_count();
    const long long per_sm = (blocks + sms - 1) / sms;
    int best = 1;
    for (int s = 2; s <= kMaxSplit && 2LL * s <= G; ++s) {
        const long long by_regs = 65536LL / (32LL * s * regs);
        const long long by_warps = 64 / s;
        if (std::min(by_regs, by_warps) >= per_sm) best = s;
    }
    return best;
}

template <int NT, int NJ>
int gemv_i8_regs() {
    static int regs = 0;
    if (regs == 0) {
        cudaFuncAttributes fa;
        regs = (cudaFuncGetAttributes(&fa, gemv_i8_kernel<NT, NJ>) == cudaSuccess && fa.numRegs > 0) ? fa.numRegs : 128;
    }
    return regs;
}

template <int B, int L, int NJ>
cudaError_t launch_pair(const GemvJobs<NJ>& jobs, const float* codebook, cudaStream_t st) {
    long long min_g = jobs.G[0];
    int max_batch = jobs.batch[0];
    for (int k = 1; k < jobs.n; ++k) {
        min_g = std::min<long long>(min_g, jobs.G[k]);
        max_batch = std::max(max_batch, jobs.batch[k]);
    }
    const long long groups = jobs.group0[jobs.n], blocks = jobs.block0[jobs.n];
    cudaError_t e = launch_pdl(rotate_x_kernel<B, L, NJ>, dim3(static_cast<unsigned>(groups)),
                               dim3(kRotThreads), 0, st, jobs, codebook);
    if (e != cudaSuccess) return e;
    if constexpr (B == 2) {
        if (max_batch <= 4) {
            const int split = gemv_split(blocks, min_g, gemv_i8_regs<1, NJ>());
            return launch_pdl(gemv_i8_kernel<1, NJ>, dim3(static_cast<unsigned>(blocks)), dim3(32 * split),
                              static_cast<size_t>(split) * 32 * sizeof(float4), st, jobs);
        }
        const int split = gemv_split(blocks, min_g, gemv_i8_regs<2, NJ>());
        return launch_pdl(gemv_i8_kernel<2, NJ>, dim3(static_cast<unsigned>(blocks)), dim3(32 * split),
                          static_cast<size_t>(split) * 32 * sizeof(float4), st, jobs);
    } else {
        const int split = gemv_split(blocks, min_g, gemv_regs<B, NJ>());
        return launch_pdl(gemv_split_kernel<B, NJ>, dim3(static_cast<unsigned>(blocks)), dim3(32 * split), 0,
                          st, jobs);
    }
}

template <int NJ>
cudaError_t launch_jobs(int bits, const GemvJobs<NJ>& jobs, const float* codebook, cudaStream_t st) {
    switch (bits) {
        case CQ_BITS_TERNARY: return launch_pair<2, 3, NJ>(jobs, codebook, st);
        case 2: return launch_pair<2, 4, NJ>(jobs, codebook, st);
        case 3: return launch_pair<3, 8, NJ>(jobs, codebook, st);
        default: return launch_pair<4, 16, NJ>(jobs, codebook, st);
    }
}

template <int NJ>
void set_job(GemvJobs<NJ>& jobs, int k, const GemvItem& it) {
    jobs.x[k] = it.x;
    jobs.packed[k] = it.packed;
    jobs.norms[k] = it.norms;
    jobs.ws[k] = static_cast<char*>(it.workspace);
    jobs.y[k] = it.y;
    jobs.rows[k] = it.sh.rows;
    jobs.cols[k] = it.sh.cols;
    jobs.G[k] = static_cast<int>(it.sh.groups_per_row);
    jobs.batch[k] = it.batch;
    jobs.group0[k + 1] = jobs.group0[k] + it.sh.groups_per_row;
    jobs.block0[k + 1] = jobs.block0[k] + (it.sh.rows + kRowsPerBlock - 1) / kRowsPerBlock;
}

// Products per batched launch pair: the job list travels in the kernel parameters.
constexpr int kGemvBatch = 256;
static_assert(sizeof(GemvJobs<kGemvBatch>) < 32000, "kernel parameter space");

}  // namespace

size_t gemv_workspace_bytes(long long cols, int batch) {
    // one block per 8 activation rows (the B operand is always padded to 8 columns)
    const long long G = (cols + kGroup - 1) / kGroup;
    const size_t bytes = frag_bytes(G) + scale_bytes(G) + sizeof(CodeTable);
    const size_t blocks = static_cast<size_t>(batch < 1 ? 1 : (batch + kBatchCols - 1) / kBatchCols);
    return (bytes + 255) / 256 * 256 * blocks;
}

cudaError_t launch_dequant_gemv(const uint8_t* packed, const uint16_t* norms, const Shape& sh,
                                int bits, const float* codebook, const uint16_t* x, int batch,
                                float* y, void* workspace, cudaStream_t stream) {
    GemvJobs<1> jobs;
    jobs.n = 1;
    jobs.group0[0] = jobs.block0[0] = 0;
    set_job(jobs, 0, GemvItem{packed, norms, sh, x, batch, y, workspace});
    return launch_jobs(bits, jobs, codebook, stream);
}

cudaError_t launch_dequant_gemv_batch(const GemvItem* items, int count, int bits,
                                      const float* codebook, cudaStream_t stream) {
    static GemvJobs<kGemvBatch> jobs;  // host staging (large); calls are serialised below
    static std::mutex mu;
    std::lock_guard<std::mutex> lock(mu);
    for (int i0 = 0; i0 < count; i0 += kGemvBatch) {
        const int n = std::min(kGemvBatch, count - i0);
        jobs.n = n;
        jobs.group0[0] = jobs.block0[0] = 0;
        for (int k = 0; k < n; ++k) set_job(jobs, k, items[i0 + k]);
        const cudaError_t e = launch_jobs(bits, jobs, codebook, stream);
        if (e != cudaSuccess) return e;
    }
    return cudaSuccess;
}

}  // namespace cq
