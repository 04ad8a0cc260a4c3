// cq_gemv.cu -- fused dequant-GEMV  y = W_hat x  without materialising W_hat.
//
// H is symmetric and orthonormal (pages "Cactus Quants CQ2-bit Quantization" and "How
// CQ2-bit Quantization Contributes to Needle 2's Small Footprint", "Hadamard Rotation"),
// so for group j of row r
//     <w_hat_rj, x_j> = <H (n_rj c[idx_rj]), x_j> = n_rj <c[idx_rj], H x_j>.
// Each activation group is rotated once; the packed weights are never expanded in memory.
//
// Step 1 (rotate_x_kernel, one block per group j, one warp per batch column b < 8):
//   x~_bj = H_int x_bj (zero for b >= batch), scaled by 2^-e_bj so its largest magnitude sits
//   in [2^13, 2^14), rounded to fp16 and written in the register-fragment order of the
//   tensor-core B operand; the exponents go to an fp32 table.  Block 0 also writes the
//   codeword table (fp16, one exact power-of-two scale) used by step 2.
//
// Step 2 (gemv_mma_kernel, launched as a programmatic dependent of step 1): a 4-warp block
// owns 16 output rows.  The packed blocks of those rows are copied to shared memory with
// cp.async before anything else (the whole tile's loads are in flight at once), then each
// warp takes every fourth group: eight m16n8k16 fp16 MMAs per group (A = decoded codewords
// of 16 rows x 16 weights, B = x~ of 16 weights x 8 columns, fp32 accumulate), folded into
// fp32 totals as  total += n_rj * 2^e_bj * acc.  The warps' totals are summed in a fixed
// order, so the output is deterministic.
//
// K order inside a group.  The MMA contracts over the 16 weights of a k-step in any order
// as long as A and B agree.  Lane (g, t) = (lane / 4, lane % 4) in k-step s takes the
// weights  e = 16 w + 4 q + p,  q = 0..3,  with  w = t + 4 (s / 4)  and  p = s % 4:  the
// four codes sitting at bit 2p of the four bytes of packed word w.  For 2-bit codes the
// decode is then an (immediate) shift, a mask, two integer multiply-adds that form
// byte-permute selectors, and two PRMTs from a 4-entry fp16 table held in two registers.
#include <algorithm>

#include "cq_device.cuh"
#include "cq_internal.h"

namespace cq {
namespace {

using namespace dev;

constexpr int kRotThreads = 256;  // 8 warps = 8 batch columns
constexpr int kRowsPerBlock = 16;
constexpr int kWarps = 4;
constexpr int kThreads = 32 * kWarps;
constexpr int kBatchCols = 8;     // MMA N: batch columns, zero padded
constexpr int kXEntry = 8;        // bytes of B fragment per lane per k-step (4 fp16)

// Workspace: [G][8 k-steps][32 lanes] of 4 fp16 | fp32 exponents [G][8] | codeword table.
size_t frag_bytes(long long G) { return static_cast<size_t>(G) * 8 * 32 * kXEntry; }
size_t scale_bytes(long long G) { return static_cast<size_t>(G) * kBatchCols * sizeof(float); }

struct CodeTable {
    uint32_t lo, hi;      // low / high bytes of the fp16 codewords 0..3 (2-bit codes)
    float inv_scale;      // 2^-cs: the table holds fp16(c_k 2^cs)
    uint32_t pad;
    uint16_t h[16];       // fp16 codewords 0..15 (entries past L repeat the last level)
};

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

__device__ __forceinline__ void mma_16816(float (&c)[4], uint32_t a0, uint32_t a1, uint32_t a2,
                                          uint32_t a3, uint32_t b0, uint32_t b1) {
    asm volatile(
        "mma.sync.aligned.m16n8k16.row.col.f32.f16.f16.f32 {%0, %1, %2, %3}, {%4, %5, %6, %7}, "
        "{%8, %9}, {%0, %1, %2, %3};"
        : "+f"(c[0]), "+f"(c[1]), "+f"(c[2]), "+f"(c[3])
        : "r"(a0), "r"(a1), "r"(a2), "r"(a3), "r"(b0), "r"(b1));
}

// ---------------------------------------------------------------------------------------
// step 1: rotate the activations into fragment order (+ codeword table)
// ---------------------------------------------------------------------------------------

template <int L>
__global__ void __launch_bounds__(kRotThreads)
    rotate_x_kernel(const uint16_t* __restrict__ x, long long cols, long long G, int batch,
                    const float* __restrict__ codebook, __half* __restrict__ xfrag,
                    float* __restrict__ xscale, CodeTable* __restrict__ table) {
    // the GEMV that follows may start its weight copies now (it waits before reading x~)
    asm volatile("griddepcontrol.launch_dependents;");
    const long long j = blockIdx.x;
    const int b = threadIdx.x >> 5, lane = threadIdx.x & 31;

    if (j == 0 && threadIdx.x < 32) {
        float m = 0.0f;
#pragma unroll
        for (int k = 0; k < L; ++k) m = fmaxf(m, fabsf(__ldg(codebook + k)));
        const int cs = (m > 0.0f) ? (13 - ilogbf(m)) : 0;
        const int k = threadIdx.x < 16 ? (threadIdx.x < L ? static_cast<int>(threadIdx.x) : L - 1) : 0;
        const uint32_t u = __half_as_ushort(__float2half_rn(ldexpf(__ldg(codebook + k), cs)));
        if (threadIdx.x < 16) table->h[threadIdx.x] = static_cast<uint16_t>(u);
        // bytes of codewords 0..3 gathered in every lane
        uint32_t lo = 0, hi = 0;
#pragma unroll
        for (int q = 0; q < 4; ++q) {
            const uint32_t uq = __shfl_sync(kFullMask, u, q);
            lo |= (uq & 0xffu) << (8 * q);
            hi |= (uq >> 8) << (8 * q);
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
    // element el = 4 lane + i = 16 w + 4 q + p  ->  k-step s = p + 4 (w / 4), lane 4 b + w % 4,
    // half q of the lane's 4-value entry
    const int w = lane >> 2, q = lane & 3;
    const int t = w & 3, shi = w >> 2;
#pragma unroll
    for (int p = 0; p < 4; ++p) {
        const int s = p + 4 * shi;
        xfrag[((j * 8 + s) * 32 + 4 * b + t) * 4 + q] = __float2half_rn(v[p] * down);
    }
}

// ---------------------------------------------------------------------------------------
// step 2: streaming tensor-core GEMV
// ---------------------------------------------------------------------------------------

__device__ __forceinline__ long long min64(long long a, long long b) { return a < b ? a : b; }

__device__ __forceinline__ void cp_async16(void* smem, const void* gmem) {
    const uint32_t d = static_cast<uint32_t>(__cvta_generic_to_shared(smem));
    asm volatile("cp.async.cg.shared.global [%0], [%1], 16;" ::"r"(d), "l"(gmem) : "memory");
}
__device__ __forceinline__ void cp_async_commit() { asm volatile("cp.async.commit_group;" ::: "memory"); }
template <int N>
__device__ __forceinline__ void cp_async_wait() { asm volatile("cp.async.wait_group %0;" ::"n"(N) : "memory"); }

// Groups are staged in chunks of kChunk; a stage holds 16 rows x kChunk blocks, each row
// padded by 16 bytes so the eight rows a warp reads at once fall in different banks.
constexpr int kChunk = 32;
constexpr int kStages = 4;

template <int B>
struct Stage {
    static constexpr int kRowBytes = kChunk * 16 * B + 16;
    static constexpr int kBytes = kRowsPerBlock * kRowBytes;
};

template <int B>
__device__ __forceinline__ void issue_chunk(const uint8_t* __restrict__ packed, long long rows,
                                            long long G, long long r0, long long j0, int len,
                                            uint8_t* stage) {
    constexpr int kFullPieces = kChunk * B;  // 16-byte pieces per row of a full chunk
    if (len == kChunk) {
        for (int i = threadIdx.x; i < kRowsPerBlock * kFullPieces; i += kThreads) {
            const int r = i / kFullPieces, p = i % kFullPieces;
            if (r0 + r < rows)
                cp_async16(stage + r * Stage<B>::kRowBytes + 16 * p,
                           packed + ((r0 + r) * G + j0) * (16 * B) + 16 * p);
        }
    } else {
        const int pieces = len * B;
        for (int i = threadIdx.x; i < kRowsPerBlock * pieces; i += kThreads) {
            const int r = i / pieces, p = i - r * pieces;
            if (r0 + r < rows)
                cp_async16(stage + r * Stage<B>::kRowBytes + 16 * p,
                           packed + ((r0 + r) * G + j0) * (16 * B) + 16 * p);
        }
    }
}

// The 16 B-bit codes lane t uses from one group row, for the halves h = 0 (k-steps 0-3) and
// h = 1 (k-steps 4-7): bits [16 B w0, 16 B w0 + 16 B) of the block with w0 = t + 4 h.
template <int B>
struct RowCodes {
    uint32_t seg[2][(B + 1) / 2];  // 1 word per half for B = 2, 2 words for B = 3, 4
};

template <int B>
__device__ __forceinline__ void load_codes(const uint8_t* row, int t, RowCodes<B>& rc) {
    const uint32_t* wd = reinterpret_cast<const uint32_t*>(row);
#pragma unroll
    for (int h = 0; h < 2; ++h) {
        const int w0 = t + 4 * h;
        if constexpr (B == 2) {
            rc.seg[h][0] = wd[w0];
        } else if constexpr (B == 4) {
            rc.seg[h][0] = wd[2 * w0];
            rc.seg[h][1] = wd[2 * w0 + 1];
        } else {
            // 48 bits at bit 48 w0: three words from word 3 w0 / 2, shifted by 16 (w0 & 1)
            const int wi = (3 * w0) >> 1;
            const uint32_t a = wd[wi], b = wd[wi + 1], c = wd[wi + 2];
            const uint32_t sh = 16u * (w0 & 1);
            rc.seg[h][0] = __funnelshift_r(a, b, sh);
            rc.seg[h][1] = __funnelshift_r(b, c, sh);
        }
    }
}

// A-fragment pair of one row in k-step s: (c[e0], c[e1]) and (c[e2], c[e3]).
template <int B>
__device__ __forceinline__ void decode(const RowCodes<B>& rc, int s, uint32_t tlo, uint32_t thi,
                                       const uint16_t* __restrict__ tab, uint32_t& r0, uint32_t& r1) {
    const int h = s >> 2, p = s & 3;
    if constexpr (B == 2) {
        const uint32_t sw = (rc.seg[h][0] >> (2 * p)) & 0x03030303u;  // code q in byte q
        r0 = prmt(tlo, thi, sw * 0x11u + 0x4040u);                  // selectors of codes 0, 1
        r1 = prmt(tlo, thi, mad_hi(sw, 0x110000u, 0x4040u));        // selectors of codes 2, 3
    } else {
        uint32_t code[4];
#pragma unroll
        for (int q = 0; q < 4; ++q) {
            const int bit = B * (4 * q + p);  // within the 16 B-bit segment
            const uint32_t lo = rc.seg[h][bit >> 5];
            const uint32_t hi = ((bit >> 5) + 1 < (B + 1) / 2) ? rc.seg[h][(bit >> 5) + 1] : 0u;
            code[q] = __funnelshift_r(lo, hi, bit & 31) & ((1u << B) - 1u);
        }
        r0 = static_cast<uint32_t>(tab[code[0]]) | (static_cast<uint32_t>(tab[code[1]]) << 16);
        r1 = static_cast<uint32_t>(tab[code[2]]) | (static_cast<uint32_t>(tab[code[3]]) << 16);
    }
}

template <int B, int NST>
__global__ void __launch_bounds__(kThreads, 8)
    gemv_mma_kernel(const uint8_t* __restrict__ packed, const uint16_t* __restrict__ norms,
                    long long rows, long long G, const uint2* __restrict__ xfrag,
                    const float* __restrict__ xscale, const CodeTable* __restrict__ table,
                    int batch, float* __restrict__ y) {
    extern __shared__ __align__(16) uint8_t smem[];  // NST stages, then NST norm tiles
    float* nrm_s = reinterpret_cast<float*>(smem + NST * Stage<B>::kBytes);
    __shared__ float4 red[kWarps][32];
    __shared__ uint16_t tab_s[16];
    constexpr int kNrm = kRowsPerBlock * kChunk;
    constexpr int kNrmPerThread = kNrm / kThreads;

    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int g = lane >> 2, t = lane & 3;
    const long long r0 = static_cast<long long>(blockIdx.x) * kRowsPerBlock;
    const long long ra = r0 + g, rb = r0 + g + 8;
    const bool oka = ra < rows, okb = rb < rows;
    const long long nchunks = (G + kChunk - 1) / kChunk;

    auto norm_at = [&](long long c, int i) -> float {  // i-th norm of chunk c ([row][jj])
        const int r = i / kChunk, jj = i % kChunk;
        const long long j = c * kChunk + jj;
        return (c < nchunks && r0 + r < rows && j < G)
                   ? __half2float(__ushort_as_half(__ldg(norms + (r0 + r) * G + j)))
                   : 0.0f;
    };

    // prologue (independent of step 1): weight copies, then norms
    for (int c = 0; c < NST; ++c) {
        if (c < nchunks) {
            const long long j0 = c * kChunk;
            issue_chunk<B>(packed, rows, G, r0, j0, static_cast<int>(min64(kChunk, G - j0)),
                           smem + c * Stage<B>::kBytes);
        }
        cp_async_commit();
    }
    {
        float tmp[NST * kNrmPerThread];
#pragma unroll
        for (int c = 0; c < NST; ++c)
#pragma unroll
            for (int q = 0; q < kNrmPerThread; ++q)
                tmp[c * kNrmPerThread + q] = norm_at(c, threadIdx.x + q * kThreads);
#pragma unroll
        for (int c = 0; c < NST; ++c)
#pragma unroll
            for (int q = 0; q < kNrmPerThread; ++q)
                nrm_s[c * kNrm + threadIdx.x + q * kThreads] = tmp[c * kNrmPerThread + q];
    }

    // the rotated activations and the codeword table come from step 1
    asm volatile("griddepcontrol.wait;" ::: "memory");
    const uint32_t tlo = table->lo, thi = table->hi;
    const float inv_scale = table->inv_scale;
    if (B != 2 && threadIdx.x < 16) tab_s[threadIdx.x] = table->h[threadIdx.x];

    float tot[4] = {0.0f, 0.0f, 0.0f, 0.0f};
    for (long long c = 0; c < nchunks; ++c) {
        const int st = static_cast<int>(c % NST);
        cp_async_wait<NST - 1>();
        __syncthreads();
        const long long j0 = c * kChunk;
        const int len = static_cast<int>(min64(kChunk, G - j0));
        const uint8_t* base = smem + st * Stage<B>::kBytes;
        const float* nst = nrm_s + st * kNrm;
        uint2 bf[8];
        if (warp < len) {
            const uint2* xf = xfrag + (j0 + warp) * 8 * 32 + lane;
#pragma unroll
            for (int s = 0; s < 8; ++s) bf[s] = __ldg(xf + s * 32);
        }
        for (int jj = warp; jj < len; jj += kWarps) {
            uint2 bn[8];  // B fragments of this warp's next group, fetched during this one
            const int jn = jj + kWarps;
            if (jn < len) {
                const uint2* xf = xfrag + (j0 + jn) * 8 * 32 + lane;
#pragma unroll
                for (int s = 0; s < 8; ++s) bn[s] = __ldg(xf + s * 32);
            }
            RowCodes<B> ca, cb;
            load_codes<B>(base + g * Stage<B>::kRowBytes + jj * 16 * B, t, ca);
            load_codes<B>(base + (g + 8) * Stage<B>::kRowBytes + jj * 16 * B, t, cb);
            const long long j = j0 + jj;
            float acc[4] = {0.0f, 0.0f, 0.0f, 0.0f};
#pragma unroll
            for (int s = 0; s < 8; ++s) {
                uint32_t a0, a1, a2, a3;
                decode<B>(ca, s, tlo, thi, tab_s, a0, a2);
                decode<B>(cb, s, tlo, thi, tab_s, a1, a3);
                mma_16816(acc, a0, a1, a2, a3, bf[s].x, bf[s].y);
            }
            const float sa = nst[g * kChunk + jj], sb = nst[(g + 8) * kChunk + jj];
            const float x0 = __ldg(xscale + j * kBatchCols + 2 * t);
            const float x1 = __ldg(xscale + j * kBatchCols + 2 * t + 1);
            tot[0] = fmaf(sa * x0, acc[0], tot[0]);
            tot[1] = fmaf(sa * x1, acc[1], tot[1]);
            tot[2] = fmaf(sb * x0, acc[2], tot[2]);
            tot[3] = fmaf(sb * x1, acc[3], tot[3]);
#pragma unroll
            for (int s = 0; s < 8; ++s) bf[s] = bn[s];
        }
        __syncthreads();  // stage st fully consumed
        const long long cn = c + NST;
        if (cn < nchunks) {
            const long long jn = cn * kChunk;
            issue_chunk<B>(packed, rows, G, r0, jn, static_cast<int>(min64(kChunk, G - jn)),
                           smem + st * Stage<B>::kBytes);
        }
        cp_async_commit();
        if (cn < nchunks) {
            float tmp[kNrmPerThread];
#pragma unroll
            for (int q = 0; q < kNrmPerThread; ++q) tmp[q] = norm_at(cn, threadIdx.x + q * kThreads);
#pragma unroll
            for (int q = 0; q < kNrmPerThread; ++q) nrm_s[st * kNrm + threadIdx.x + q * kThreads] = tmp[q];
        }
    }
    cp_async_wait<0>();
    red[warp][lane] = make_float4(tot[0], tot[1], tot[2], tot[3]);
    __syncthreads();
    if (warp == 0) {
        float4 a = red[0][lane];
#pragma unroll
        for (int w = 1; w < kWarps; ++w) {
            const float4 b = red[w][lane];
            a.x += b.x;
            a.y += b.y;
            a.z += b.z;
            a.w += b.w;
        }
        const float f = inv_scale * kInvSqrt128;
        const int c0 = 2 * t, c1 = 2 * t + 1;
        if (oka && c0 < batch) y[c0 * rows + ra] = a.x * f;
        if (oka && c1 < batch) y[c1 * rows + ra] = a.y * f;
        if (okb && c0 < batch) y[c0 * rows + rb] = a.z * f;
        if (okb && c1 < batch) y[c1 * rows + rb] = a.w * f;
    }
}

template <int B, int NST>
cudaError_t launch_gemv_cfg(const uint8_t* packed, const uint16_t* norms, const Shape& sh,
                            const uint2* xfrag, const float* xscale, const CodeTable* table,
                            int batch, float* y, cudaStream_t st) {
    const long long blocks = (sh.rows + kRowsPerBlock - 1) / kRowsPerBlock;
    const int smem = NST * (Stage<B>::kBytes + kRowsPerBlock * kChunk * static_cast<int>(sizeof(float)));
    int dev = 0;
    cudaError_t e = cudaGetDevice(&dev);
    if (e != cudaSuccess) return e;
    static unsigned long long configured = 0;  // one bit per device (function attributes are per device)
    const unsigned long long bit = 1ull << (dev & 63);
    if (!(configured & bit)) {
        e = cudaFuncSetAttribute(gemv_mma_kernel<B, NST>, cudaFuncAttributeMaxDynamicSharedMemorySize, smem);
        if (e != cudaSuccess) return e;
        configured |= bit;
    }
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = dim3(static_cast<unsigned>(blocks));
    cfg.blockDim = dim3(kThreads);
    cfg.dynamicSmemBytes = static_cast<size_t>(smem);
    cfg.stream = st;
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    attr[0].val.programmaticStreamSerializationAllowed = 1;
    cfg.attrs = attr;
    cfg.numAttrs = 1;
    return cudaLaunchKernelEx(&cfg, gemv_mma_kernel<B, NST>, packed, norms, sh.rows, sh.groups_per_row,
                              xfrag, xscale, table, batch, y);
}

template <int B>
cudaError_t launch_gemv_bits(const uint8_t* packed, const uint16_t* norms, const Shape& sh,
                             const uint2* xfrag, const float* xscale, const CodeTable* table,
                             int batch, float* y, cudaStream_t st) {
    const long long nchunks = (sh.groups_per_row + kChunk - 1) / kChunk;
    if (nchunks <= 1) return launch_gemv_cfg<B, 1>(packed, norms, sh, xfrag, xscale, table, batch, y, st);
    if (nchunks == 2) return launch_gemv_cfg<B, 2>(packed, norms, sh, xfrag, xscale, table, batch, y, st);
    return launch_gemv_cfg<B, kStages>(packed, norms, sh, xfrag, xscale, table, batch, y, st);
}

template <int L>
cudaError_t launch_rotate(const uint16_t* x, const Shape& sh, int batch, const float* codebook,
                          __half* xfrag, float* xscale, CodeTable* table, cudaStream_t st) {
    rotate_x_kernel<L><<<static_cast<unsigned>(sh.groups_per_row), kRotThreads, 0, st>>>(
        x, sh.cols, sh.groups_per_row, batch, codebook, xfrag, xscale, table);
    return cudaGetLastError();
}

}  // namespace

size_t gemv_workspace_bytes(long long cols, int batch) {
    (void)batch;  // the B operand is always padded to 8 columns
    const long long G = (cols + kGroup - 1) / kGroup;
    const size_t bytes = frag_bytes(G) + scale_bytes(G) + sizeof(CodeTable);
    return (bytes + 255) / 256 * 256;
}

cudaError_t launch_dequant_gemv(const uint8_t* packed, const uint16_t* norms, const Shape& sh,
                                int bits, const float* codebook, const uint16_t* x, int batch,
                                float* y, void* workspace, cudaStream_t stream) {
    const long long G = sh.groups_per_row;
    char* ws = static_cast<char*>(workspace);
    __half* xfrag = reinterpret_cast<__half*>(ws);
    float* xscale = reinterpret_cast<float*>(ws + frag_bytes(G));
    CodeTable* table = reinterpret_cast<CodeTable*>(ws + frag_bytes(G) + scale_bytes(G));
    const uint2* xf = reinterpret_cast<const uint2*>(xfrag);
    cudaError_t e;
    switch (bits) {
        case CQ_BITS_TERNARY:
            e = launch_rotate<3>(x, sh, batch, codebook, xfrag, xscale, table, stream);
            return e != cudaSuccess ? e : launch_gemv_bits<2>(packed, norms, sh, xf, xscale, table, batch, y, stream);
        case 2:
            e = launch_rotate<4>(x, sh, batch, codebook, xfrag, xscale, table, stream);
            return e != cudaSuccess ? e : launch_gemv_bits<2>(packed, norms, sh, xf, xscale, table, batch, y, stream);
        case 3:
            e = launch_rotate<8>(x, sh, batch, codebook, xfrag, xscale, table, stream);
            return e != cudaSuccess ? e : launch_gemv_bits<3>(packed, norms, sh, xf, xscale, table, batch, y, stream);
        default:
            e = launch_rotate<16>(x, sh, batch, codebook, xfrag, xscale, table, stream);
            return e != cudaSuccess ? e : launch_gemv_bits<4>(packed, norms, sh, xf, xscale, table, batch, y, stream);
    }
}

}  // namespace cq
