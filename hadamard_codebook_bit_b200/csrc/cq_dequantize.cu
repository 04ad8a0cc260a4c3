// cq_dequantize.cu -- packed indices + fp16 norms -> W_hat (bf16 / fp32).
//
// Page "Cactus Quants CQ2-bit Quantization", "The CQ2-bit Implementation Pipeline" steps
// 5-6, and page "How Needle 2 Compresses to a Single Binary", "Stage 3" (the runtime
// rebuilds the 2-bit tensors on the fly).  Per group:
//   q_i   = c[idx_i]        (codes >= L read as the last level)
//   w_hat = H (n q) = (n / sqrt(128)) * H_int q,  n = fp32(stored fp16 norm)
//   columns >= cols are dropped.
// Same quad layout and persistent grid as the quantiser; the codebook sits in shared
// memory for the per-element lookup.
#include <algorithm>

#include "cq_device.cuh"
#include "cq_internal.h"

namespace cq {
namespace {

using namespace dev;

constexpr int kThreads = 256;
constexpr int kWarpsPerBlock = kThreads / 32;

enum Mode : int { kFlat = 0, kVector = 1, kScalar = 2 };

// Field bits of the chunk c = 4k + s (8 indices = B bytes at byte offset c * B).
template <int B>
__device__ __forceinline__ uint32_t load_chunk_bits(const uint8_t* __restrict__ blk, int c) {
    if constexpr (B == 2) {
        return __ldg(reinterpret_cast<const uint16_t*>(blk) + c);
    } else if constexpr (B == 4) {
        return __ldg(reinterpret_cast<const uint32_t*>(blk) + c);
    } else {
        const uint8_t* p = blk + 3 * c;
        return static_cast<uint32_t>(__ldg(p)) | (static_cast<uint32_t>(__ldg(p + 1)) << 8) |
               (static_cast<uint32_t>(__ldg(p + 2)) << 16);
    }
}

template <bool kBF16, int kMode>
__device__ __forceinline__ void store_group(void* __restrict__ out, long long row, long long j,
                                            long long gid, long long cols, int s,
                                            const float (&v)[kValsPerThread], float scale) {
    const long long base = (kMode == kFlat) ? gid * 128 : row * cols + j * 128;
    const long long col0 = j * 128;
#pragma unroll
    for (int k = 0; k < 4; ++k) {
        const int e0 = 32 * k + 8 * s;
        if constexpr (kMode == kScalar) {
#pragma unroll
            for (int i = 0; i < 8; ++i) {
                if (col0 + e0 + i < cols) {
                    const float x = v[8 * k + i] * scale;
                    if constexpr (kBF16)
                        static_cast<__nv_bfloat16*>(out)[base + e0 + i] = __float2bfloat16_rn(x);
                    else
                        static_cast<float*>(out)[base + e0 + i] = x;
                }
            }
        } else if constexpr (kBF16) {
            if (kMode == kFlat || col0 + e0 < cols) {
                uint4 o;
                o.x = pack_bf16x2(v[8 * k + 0] * scale, v[8 * k + 1] * scale);
                o.y = pack_bf16x2(v[8 * k + 2] * scale, v[8 * k + 3] * scale);
                o.z = pack_bf16x2(v[8 * k + 4] * scale, v[8 * k + 5] * scale);
                o.w = pack_bf16x2(v[8 * k + 6] * scale, v[8 * k + 7] * scale);
                st_stream16(static_cast<uint16_t*>(out) + base + e0, o);
            }
        } else {
#pragma unroll
            for (int h = 0; h < 2; ++h) {
                if (kMode == kFlat || col0 + e0 + 4 * h < cols) {
                    uint4 o;
                    o.x = __float_as_uint(v[8 * k + 4 * h + 0] * scale);
                    o.y = __float_as_uint(v[8 * k + 4 * h + 1] * scale);
                    o.z = __float_as_uint(v[8 * k + 4 * h + 2] * scale);
                    o.w = __float_as_uint(v[8 * k + 4 * h + 3] * scale);
                    st_stream16(static_cast<float*>(out) + base + e0 + 4 * h, o);
                }
            }
        }
    }
}

template <int B, int L, bool kBF16, int kMode>
__global__ void __launch_bounds__(kThreads)
    dequantize_kernel(const uint8_t* __restrict__ packed, const uint16_t* __restrict__ norms,
                      long long cols, long long G, long long total,
                      const float* __restrict__ codebook, void* __restrict__ out) {
    __shared__ float cb_s[16];
    pdl_trigger();
    pdl_wait();
    if (threadIdx.x < 16) cb_s[threadIdx.x] = threadIdx.x < L ? codebook[threadIdx.x] : 0.0f;
    __syncthreads();

    const int lane = threadIdx.x & 31;
    const int q = lane >> 2, s = lane & 3;
    const long long warp0 = static_cast<long long>(blockIdx.x) * kWarpsPerBlock + (threadIdx.x >> 5);
    const long long wstride = static_cast<long long>(gridDim.x) * kWarpsPerBlock;
    constexpr int kBlkBytes = 16 * B;
    constexpr uint32_t kMask = (1u << B) - 1u;

    for (long long wg = warp0 * kGroupsPerWarp; wg < total; wg += wstride * kGroupsPerWarp) {
        const long long gid = wg + q;
        const bool valid = gid < total;
        float v[kValsPerThread];
        float scale = 0.0f;
        if (valid) {
            const uint8_t* blk = packed + gid * kBlkBytes;
#pragma unroll
            for (int k = 0; k < 4; ++k) {
                const uint32_t p = load_chunk_bits<B>(blk, 4 * k + s);
#pragma unroll
                for (int i = 0; i < 8; ++i) {
                    uint32_t idx = (p >> (B * i)) & kMask;
                    if constexpr (L < (1 << B)) idx = min(idx, static_cast<uint32_t>(L - 1));
                    v[8 * k + i] = cb_s[idx];
                }
            }
            scale = __half2float(__ushort_as_half(__ldg(norms + gid))) * kInvSqrt128;
        } else {
#pragma unroll
            for (int t = 0; t < kValsPerThread; ++t) v[t] = 0.0f;
        }

        fwht128(v, s);

        if (valid) {
            long long row = 0, j = 0;
            if (kMode != kFlat) {
                row = gid / G;
                j = gid - row * G;
            }
            store_group<kBF16, kMode>(out, row, j, gid, cols, s, v, scale);
        }
    }
}

template <int B, int L, bool kBF16>
cudaError_t launch_mode(int mode, const uint8_t* packed, const uint16_t* norms, const Shape& sh,
                        const float* cb, void* out, cudaStream_t st) {
    const long long warps_needed = (sh.total_groups + kGroupsPerWarp - 1) / kGroupsPerWarp;
    const long long blocks_needed = (warps_needed + kWarpsPerBlock - 1) / kWarpsPerBlock;
    const int max_blocks = sm_count() * (2048 / kThreads);
    const int grid = static_cast<int>(std::max<long long>(1, std::min<long long>(blocks_needed, max_blocks)));
    switch (mode) {
        case kFlat:
            return launch_pdl(dequantize_kernel<B, L, kBF16, kFlat>, dim3(grid), dim3(kThreads), 0, st,
                              packed, norms, sh.cols, sh.groups_per_row, sh.total_groups, cb, out);
        case kVector:
            return launch_pdl(dequantize_kernel<B, L, kBF16, kVector>, dim3(grid), dim3(kThreads), 0, st,
                              packed, norms, sh.cols, sh.groups_per_row, sh.total_groups, cb, out);
        default:
            return launch_pdl(dequantize_kernel<B, L, kBF16, kScalar>, dim3(grid), dim3(kThreads), 0, st,
                              packed, norms, sh.cols, sh.groups_per_row, sh.total_groups, cb, out);
    }
}

template <int B, int L>
cudaError_t launch_dtype(int out_dtype, int mode, const uint8_t* packed, const uint16_t* norms,
                         const Shape& sh, const float* cb, void* out, cudaStream_t st) {
    if (out_dtype == CQ_BF16) return launch_mode<B, L, true>(mode, packed, norms, sh, cb, out, st);
    return launch_mode<B, L, false>(mode, packed, norms, sh, cb, out, st);
}

}  // namespace

cudaError_t launch_dequantize(const uint8_t* packed, const uint16_t* norms, const Shape& sh,
                              int bits, const float* codebook, void* out, int out_dtype,
                              cudaStream_t stream) {
    if (tcgen05_enabled() && dequantize_tc_supported(out_dtype, sh)) {
        unsigned* status = device_status_ptr();
        if (status != nullptr)
            return launch_dequantize_tc(packed, norms, sh, bits, codebook, out, out_dtype, status, stream);
    }
    const int chunk = (out_dtype == CQ_BF16) ? 8 : 4;
    const int mode = (sh.cols % 128 == 0) ? kFlat : (sh.cols % chunk == 0) ? kVector : kScalar;
    switch (bits) {
        case CQ_BITS_TERNARY:
            return launch_dtype<2, 3>(out_dtype, mode, packed, norms, sh, codebook, out, stream);
        case 2:
            return launch_dtype<2, 4>(out_dtype, mode, packed, norms, sh, codebook, out, stream);
        case 3:
            return launch_dtype<3, 8>(out_dtype, mode, packed, norms, sh, codebook, out, stream);
        default:
            return launch_dtype<4, 16>(out_dtype, mode, packed, norms, sh, codebook, out, stream);
    }
}

}  // namespace cq
