// cq_quantize.cu -- W (bf16 / fp32) -> packed indices + fp16 norms.
//
// Page "Cactus Quants CQ2-bit Quantization", "The CQ2-bit Implementation Pipeline" steps
// 1-4, stored as page "How CQ2-bit Quantization Contributes to Needle 2's Small Footprint",
// "Per-Group Storage Breakdown" / "Binary Serialization" describe.  Per group:
//   v   = the 128 elements, zero padded past cols          (step 1)
//   r   = H_int v  (H_int = sqrt(128) H, +-1 entries)        (step 2)
//   n   = ||H v|| = sqrt(sum r^2 / 128), stored fp16 RNE     (step 3)
//   idx = #{k : r > m_k * ||r||} with m_k the fp32 midpoints of consecutive codewords,
//         i.e. the nearest codeword of u = r / ||r|| with ties to the lower index; when
//         the group is all zero, u = 0 and idx = #{k : 0 > m_k}    (step 4)
//   indices packed LSB first, b bits each.
//
// HBM-bound streaming kernel: a persistent grid of 256-thread blocks, each warp takes
// eight groups per iteration (one per quad, see cq_device.cuh), no shared memory.
#include <algorithm>

#include "cq_device.cuh"
#include "cq_internal.h"

namespace cq {
namespace {

using namespace dev;

constexpr int kThreads = 256;
constexpr int kWarpsPerBlock = kThreads / 32;

// How a kernel addresses its groups.
enum Mode : int {
    kFlat = 0,    // cols % 128 == 0: group g starts at element 128 g, never padded
    kVector = 1,  // rows start on 16-byte boundaries; the last group of a row may be short
    kScalar = 2   // anything else: element-wise loads with bounds checks
};

template <bool kBF16, int kMode>
__device__ __forceinline__ void load_group(const void* __restrict__ w, long long row, long long j,
                                           long long gid, long long cols, int s, bool valid,
                                           float (&v)[kValsPerThread]) {
#pragma unroll
    for (int t = 0; t < kValsPerThread; ++t) v[t] = 0.0f;
    if (!valid) return;
    const long long base = (kMode == kFlat) ? gid * 128 : row * cols + j * 128;
    const long long col0 = j * 128;  // first column of the group (unused in flat mode)
#pragma unroll
    for (int k = 0; k < 4; ++k) {
        const int e0 = 32 * k + 8 * s;  // first element of this thread's chunk
        if constexpr (kMode == kScalar) {
#pragma unroll
            for (int i = 0; i < 8; ++i) {
                if (col0 + e0 + i < cols) {
                    if constexpr (kBF16)
                        v[8 * k + i] = bf16_bits_to_float(
                            static_cast<const uint16_t*>(w)[base + e0 + i]);
                    else
                        v[8 * k + i] = static_cast<const float*>(w)[base + e0 + i];
                }
            }
        } else if constexpr (kBF16) {
            if (kMode == kFlat || col0 + e0 < cols) {  // cols % 8 == 0: chunk all-in or all-out
                const uint4 q = ld_stream16(static_cast<const uint16_t*>(w) + base + e0);
                v[8 * k + 0] = bf16_lo(q.x);
                v[8 * k + 1] = bf16_hi(q.x);
                v[8 * k + 2] = bf16_lo(q.y);
                v[8 * k + 3] = bf16_hi(q.y);
                v[8 * k + 4] = bf16_lo(q.z);
                v[8 * k + 5] = bf16_hi(q.z);
                v[8 * k + 6] = bf16_lo(q.w);
                v[8 * k + 7] = bf16_hi(q.w);
            }
        } else {
#pragma unroll
            for (int h = 0; h < 2; ++h) {  // two 16-byte halves of four fp32 each
                if (kMode == kFlat || col0 + e0 + 4 * h < cols) {
                    const uint4 q =
                        ld_stream16(static_cast<const float*>(w) + base + e0 + 4 * h);
                    v[8 * k + 4 * h + 0] = __uint_as_float(q.x);
                    v[8 * k + 4 * h + 1] = __uint_as_float(q.y);
                    v[8 * k + 4 * h + 2] = __uint_as_float(q.z);
                    v[8 * k + 4 * h + 3] = __uint_as_float(q.w);
                }
            }
        }
    }
}

template <int B, int L, bool kBF16, int kMode>
__global__ void __launch_bounds__(kThreads)
    quantize_kernel(const void* __restrict__ w, long long cols, long long G, long long total,
                    const float* __restrict__ codebook, uint8_t* __restrict__ packed,
                    uint16_t* __restrict__ norms) {
    pdl_trigger();
    pdl_wait();
    const int lane = threadIdx.x & 31;
    const int q = lane >> 2, s = lane & 3;

    // fp32 decision midpoints between consecutive codewords
    float mid[L - 1];
#pragma unroll
    for (int k = 0; k < L - 1; ++k) mid[k] = 0.5f * (__ldg(codebook + k) + __ldg(codebook + k + 1));

    const long long warp0 = static_cast<long long>(blockIdx.x) * kWarpsPerBlock + (threadIdx.x >> 5);
    const long long wstride = static_cast<long long>(gridDim.x) * kWarpsPerBlock;
    constexpr int kBlkBytes = 16 * B;  // 128 indices * B bits

    for (long long wg = warp0 * kGroupsPerWarp; wg < total; wg += wstride * kGroupsPerWarp) {
        const long long gid = wg + q;
        const bool valid = gid < total;
        long long row = 0, j = 0;
        if (kMode != kFlat) {
            row = gid / G;
            j = gid - row * G;
        }
        float v[kValsPerThread];
        load_group<kBF16, kMode>(w, row, j, gid, cols, s, valid, v);

        fwht128(v, s);

        float ss = 0.0f;
#pragma unroll
        for (int t = 0; t < kValsPerThread; ++t) ss = fmaf(v[t], v[t], ss);
        ss = quad_sum(ss);
        const float nrm = sqrtf(ss);  // ||H_int v|| = sqrt(128) * n
        float T[L - 1];
#pragma unroll
        for (int k = 0; k < L - 1; ++k) T[k] = nrm > 0.0f ? mid[k] * nrm : mid[k];

        uint8_t* blk = packed + gid * kBlkBytes;
#pragma unroll
        for (int k = 0; k < 4; ++k) {
            uint32_t p = 0;
#pragma unroll
            for (int i = 0; i < 8; ++i) p |= nearest_index<L>(v[8 * k + i], T) << (B * i);
            // chunk c = 4k + s owns bytes [c*B, c*B + B) of the group block
            if constexpr (B == 2) {
                if (valid) reinterpret_cast<uint16_t*>(blk)[4 * k + s] = static_cast<uint16_t>(p);
            } else if constexpr (B == 4) {
                if (valid) reinterpret_cast<uint32_t*>(blk)[4 * k + s] = p;
            } else {
                // the quad's four 24-bit pieces form three aligned words at bytes 12k..12k+11
                const uint32_t nxt = __shfl_down_sync(kFullMask, p, 1);
                if (valid && s < 3)
                    reinterpret_cast<uint32_t*>(blk)[3 * k + s] =
                        (p >> (8 * s)) | (nxt << (24 - 8 * s));
            }
        }
        if (valid && s == 0) norms[gid] = __half_as_ushort(__float2half_rn(sqrtf(ss * 0.0078125f)));
    }
}

template <int B, int L, bool kBF16>
cudaError_t launch_mode(int mode, const void* w, const Shape& sh, const float* cb,
                        uint8_t* packed, uint16_t* norms, cudaStream_t st) {
    const long long warps_needed = (sh.total_groups + kGroupsPerWarp - 1) / kGroupsPerWarp;
    const long long blocks_needed = (warps_needed + kWarpsPerBlock - 1) / kWarpsPerBlock;
    const int max_blocks = sm_count() * (2048 / kThreads);
    const int grid = static_cast<int>(std::max<long long>(1, std::min<long long>(blocks_needed, max_blocks)));
    switch (mode) {
        case kFlat:
            return launch_pdl(quantize_kernel<B, L, kBF16, kFlat>, dim3(grid), dim3(kThreads), 0, st,
                              w, sh.cols, sh.groups_per_row, sh.total_groups, cb, packed, norms);
        case kVector:
            return launch_pdl(quantize_kernel<B, L, kBF16, kVector>, dim3(grid), dim3(kThreads), 0, st,
                              w, sh.cols, sh.groups_per_row, sh.total_groups, cb, packed, norms);
        default:
            return launch_pdl(quantize_kernel<B, L, kBF16, kScalar>, dim3(grid), dim3(kThreads), 0, st,
                              w, sh.cols, sh.groups_per_row, sh.total_groups, cb, packed, norms);
    }
}

template <int B, int L>
cudaError_t launch_dtype(int w_dtype, int mode, const void* w, const Shape& sh, const float* cb,
                         uint8_t* packed, uint16_t* norms, cudaStream_t st) {
    if (w_dtype == CQ_BF16) return launch_mode<B, L, true>(mode, w, sh, cb, packed, norms, st);
    return launch_mode<B, L, false>(mode, w, sh, cb, packed, norms, st);
}

}  // namespace

cudaError_t launch_quantize(const void* w, int w_dtype, const Shape& sh, int bits,
                            const float* codebook, uint8_t* packed, uint16_t* norms,
                            cudaStream_t stream) {
    if (tcgen05_enabled() && quantize_tc_supported(w_dtype, sh)) {
        unsigned* status = device_status_ptr();
        if (status != nullptr)
            return launch_quantize_tc(w, sh, bits, codebook, packed, norms, status, stream);
    }
    const int chunk = (w_dtype == CQ_BF16) ? 8 : 4;  // elements per 16 bytes
    const int mode = (sh.cols % 128 == 0) ? kFlat : (sh.cols % chunk == 0) ? kVector : kScalar;
    switch (bits) {
        case CQ_BITS_TERNARY:
            return launch_dtype<2, 3>(w_dtype, mode, w, sh, codebook, packed, norms, stream);
        case 2:
            return launch_dtype<2, 4>(w_dtype, mode, w, sh, codebook, packed, norms, stream);
        case 3:
            return launch_dtype<3, 8>(w_dtype, mode, w, sh, codebook, packed, norms, stream);
        default:
            return launch_dtype<4, 16>(w_dtype, mode, w, sh, codebook, packed, norms, stream);
    }
}

}  // namespace cq
