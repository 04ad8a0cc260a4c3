// cq_gemv.cu -- fused dequant-GEMV  y = W_hat x  without materialising W_hat.
//
// H is symmetric and orthonormal (pages "Cactus Quants CQ2-bit Quantization" and "How
// CQ2-bit Quantization Contributes to Needle 2's Small Footprint", "Hadamard Rotation"),
// so for the group j of row r
//     <w_hat_rj, x_j> = <H (n_rj c[idx_rj]), x_j> = n_rj <c[idx_rj], H x_j>.
// Step 1 rotates every activation group once (x~ = H_int x, fp32, into the workspace);
// step 2 streams the packed weights and accumulates
//     y[b, r] = (1/sqrt(128)) sum_j n_rj sum_i c[idx_rji] x~_bji      (fp32).
// The packed index stream is the only large read: b/8 + 2/128 bytes per weight.
#include <algorithm>

#include "cq_device.cuh"
#include "cq_internal.h"

namespace cq {
namespace {

using namespace dev;

constexpr int kRotThreads = 256;
constexpr int kGemvThreads = 256;

// x~[b][j][e] = (H_int x_bj)[e], natural element order, zero padded input.
__global__ void __launch_bounds__(kRotThreads)
    rotate_x_kernel(const uint16_t* __restrict__ x, long long cols, long long G, int batch,
                    float* __restrict__ xt) {
    const int lane = threadIdx.x & 31;
    const int q = lane >> 2, s = lane & 3;
    const long long total = static_cast<long long>(batch) * G;
    const long long warp0 = static_cast<long long>(blockIdx.x) * (kRotThreads / 32) + (threadIdx.x >> 5);
    const long long wstride = static_cast<long long>(gridDim.x) * (kRotThreads / 32);
    for (long long wg = warp0 * kGroupsPerWarp; wg < total; wg += wstride * kGroupsPerWarp) {
        const long long gid = wg + q;  // = b * G + j
        const bool valid = gid < total;
        const long long b = valid ? gid / G : 0, j = valid ? gid - b * G : 0;
        float v[kValsPerThread];
#pragma unroll
        for (int k = 0; k < 4; ++k) {
#pragma unroll
            for (int i = 0; i < 8; ++i) {
                const long long col = j * 128 + 32 * k + 8 * s + i;
                v[8 * k + i] = (valid && col < cols) ? bf16_bits_to_float(__ldg(x + b * cols + col)) : 0.0f;
            }
        }
        fwht128(v, s);
        if (valid) {
            float* dst = xt + gid * 128;
#pragma unroll
            for (int k = 0; k < 4; ++k) {
                float4* d = reinterpret_cast<float4*>(dst + 32 * k + 8 * s);
                d[0] = make_float4(v[8 * k + 0], v[8 * k + 1], v[8 * k + 2], v[8 * k + 3]);
                d[1] = make_float4(v[8 * k + 4], v[8 * k + 5], v[8 * k + 6], v[8 * k + 7]);
            }
        }
    }
}

// One warp per output row; lane l covers elements 4l..4l+3 of every group.
template <int B, int L, int NB>
__global__ void __launch_bounds__(kGemvThreads)
    gemv_kernel(const uint8_t* __restrict__ packed, const uint16_t* __restrict__ norms,
                long long rows, long long G, const float* __restrict__ codebook,
                const float* __restrict__ xt, float* __restrict__ y) {
    __shared__ float cb_s[16];
    if (threadIdx.x < 16) cb_s[threadIdx.x] = threadIdx.x < L ? codebook[threadIdx.x] : 0.0f;
    __syncthreads();
    const int lane = threadIdx.x & 31;
    constexpr int kBlkBytes = 16 * B;
    constexpr uint32_t kMask = (1u << B) - 1u;
    const long long warp0 = static_cast<long long>(blockIdx.x) * (kGemvThreads / 32) + (threadIdx.x >> 5);
    const long long wstride = static_cast<long long>(gridDim.x) * (kGemvThreads / 32);

    for (long long r = warp0; r < rows; r += wstride) {
        float acc[NB];
#pragma unroll
        for (int b = 0; b < NB; ++b) acc[b] = 0.0f;
        for (long long j = 0; j < G; ++j) {
            const long long gid = r * G + j;
            const uint8_t* blk = packed + gid * kBlkBytes;
            // 4B bits of this lane's four indices, starting at bit 4*B*lane
            const int bit0 = 4 * B * lane;
            const uint32_t* wp = reinterpret_cast<const uint32_t*>(blk);
            uint32_t lo = __ldg(wp + (bit0 >> 5));
            const int sh = bit0 & 31;
            uint32_t p = lo >> sh;
            if (sh + 4 * B > 32) p |= __ldg(wp + (bit0 >> 5) + 1) << (32 - sh);
            const float n = __half2float(__ushort_as_half(__ldg(norms + gid)));
            float c[4];
#pragma unroll
            for (int t = 0; t < 4; ++t) {
                uint32_t idx = (p >> (B * t)) & kMask;
                if constexpr (L < (1 << B)) idx = min(idx, static_cast<uint32_t>(L - 1));
                c[t] = cb_s[idx];
            }
#pragma unroll
            for (int b = 0; b < NB; ++b) {
                const float4 xv = __ldg(reinterpret_cast<const float4*>(xt + (b * G + j) * 128) + lane);
                float d = c[0] * xv.x;
                d = fmaf(c[1], xv.y, d);
                d = fmaf(c[2], xv.z, d);
                d = fmaf(c[3], xv.w, d);
                acc[b] = fmaf(n, d, acc[b]);
            }
        }
#pragma unroll
        for (int b = 0; b < NB; ++b) {
            float a = acc[b];
#pragma unroll
            for (int m = 16; m >= 1; m >>= 1) a += __shfl_xor_sync(kFullMask, a, m);
            if (lane == 0) y[b * rows + r] = a * kInvSqrt128;
        }
    }
}

template <int B, int L>
cudaError_t launch_gemv_bits(int batch, const uint8_t* packed, const uint16_t* norms,
                             const Shape& sh, const float* cb, const float* xt, float* y,
                             cudaStream_t st) {
    const long long blocks_needed = (sh.rows + (kGemvThreads / 32) - 1) / (kGemvThreads / 32);
    const int grid = static_cast<int>(std::max<long long>(
        1, std::min<long long>(blocks_needed, static_cast<long long>(sm_count()) * 8)));
#define CQ_GEMV_CASE(NBV)                                                                  \
    case NBV:                                                                              \
        gemv_kernel<B, L, NBV><<<grid, kGemvThreads, 0, st>>>(packed, norms, sh.rows,      \
                                                              sh.groups_per_row, cb, xt, y); \
        break;
    switch (batch) {
        CQ_GEMV_CASE(1)
        CQ_GEMV_CASE(2)
        CQ_GEMV_CASE(3)
        CQ_GEMV_CASE(4)
        CQ_GEMV_CASE(5)
        CQ_GEMV_CASE(6)
        CQ_GEMV_CASE(7)
        CQ_GEMV_CASE(8)
        default:
            return cudaErrorInvalidValue;
    }
#undef CQ_GEMV_CASE
    return cudaGetLastError();
}

}  // namespace

size_t gemv_workspace_bytes(long long cols, int batch) {
    const long long G = (cols + kGroup - 1) / kGroup;
    const size_t bytes = static_cast<size_t>(batch) * static_cast<size_t>(G) * kGroup * sizeof(float);
    return (bytes + 255) / 256 * 256;
}

cudaError_t launch_dequant_gemv(const uint8_t* packed, const uint16_t* norms, const Shape& sh,
                                int bits, const float* codebook, const uint16_t* x, int batch,
                                float* y, void* workspace, cudaStream_t stream) {
    float* xt = static_cast<float*>(workspace);
    const long long rot_groups = static_cast<long long>(batch) * sh.groups_per_row;
    const long long rot_blocks = (rot_groups + 63) / 64;
    const int rgrid = static_cast<int>(std::max<long long>(1, std::min<long long>(rot_blocks, sm_count() * 8LL)));
    rotate_x_kernel<<<rgrid, kRotThreads, 0, stream>>>(x, sh.cols, sh.groups_per_row, batch, xt);
    cudaError_t e = cudaGetLastError();
    if (e != cudaSuccess) return e;
    switch (bits) {
        case CQ_BITS_TERNARY:
            return launch_gemv_bits<2, 3>(batch, packed, norms, sh, codebook, xt, y, stream);
        case 2:
            return launch_gemv_bits<2, 4>(batch, packed, norms, sh, codebook, xt, y, stream);
        case 3:
            return launch_gemv_bits<3, 8>(batch, packed, norms, sh, codebook, xt, y, stream);
        default:
            return launch_gemv_bits<4, 16>(batch, packed, norms, sh, codebook, xt, y, stream);
    }
}

}  // namespace cq
