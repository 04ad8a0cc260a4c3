// cq_device.cuh -- device building blocks shared by the libcq kernels.
//
// Thread layout used by every group kernel: four lanes ("a quad") own one 128-element
// group, eight groups per warp.  Lane (q, s) with q = lane / 4 and s = lane % 4 holds 32
// values in registers; register j = 8k + i (k in [0,4), i in [0,8)) is element
//     e = 32k + 8s + i
// of the group.  A 16-byte bf16 load therefore brings elements 8c..8c+7 of chunk
// c = 4k + s, so the quad reads 64 contiguous bytes per k and the warp touches eight
// 256-byte groups per instruction, every sector fully used.
//
// The Sylvester Walsh-Hadamard transform factorises over the bits of e (pages "Cactus
// Quants CQ2-bit Quantization" and "How CQ2-bit Quantization Contributes to Needle 2's
// Small Footprint", "Hadamard Rotation": an orthonormal, parameter-free transform whose
// product form gives the O(N log N) fast transform).  Bits 0-2 and 5-6 of e live inside a
// thread (5 butterfly stages on registers), bits 3-4 across the quad (2 shuffle stages).
// The kernels apply the unnormalised +-1 matrix H_int = sqrt(128) H and fold 1/sqrt(128)
// into the norm / output scale.
#pragma once

#include <cstdint>

#include <cuda_bf16.h>
#include <cuda_fp16.h>
#include <cuda_runtime.h>

namespace cq {
namespace dev {

constexpr unsigned kFullMask = 0xffffffffu;
constexpr int kValsPerThread = 32;
constexpr int kGroupsPerWarp = 8;
constexpr float kInvSqrt128 = 0.088388347648318440550f;  // fp32(1/sqrt(128))

// ---------------------------------------------------------------------------------------
// programmatic dependent launch (see launch_pdl)
// ---------------------------------------------------------------------------------------

// Let the next kernel in the stream be scheduled; it still waits for this one to finish
// before touching global memory.
__device__ __forceinline__ void pdl_trigger() { asm volatile("griddepcontrol.launch_dependents;" ::: "memory"); }

// Wait until the previous kernel in the stream has finished and its writes are visible.
__device__ __forceinline__ void pdl_wait() { asm volatile("griddepcontrol.wait;" ::: "memory"); }

// ---------------------------------------------------------------------------------------
// memory helpers
// ---------------------------------------------------------------------------------------

// 16-byte streaming load that bypasses L1 allocation (inputs are read exactly once).
__device__ __forceinline__ uint4 ld_stream16(const void* p) {
    uint4 r;
    asm volatile("ld.global.nc.L1::no_allocate.v4.u32 {%0, %1, %2, %3}, [%4];"
                 : "=r"(r.x), "=r"(r.y), "=r"(r.z), "=r"(r.w)
                 : "l"(p));
    return r;
}

// 16-byte store with an evict-first hint (outputs are not re-read by this kernel).
__device__ __forceinline__ void st_stream16(void* p, uint4 v) {
    asm volatile("st.global.cs.v4.u32 [%0], {%1, %2, %3, %4};" ::"l"(p), "r"(v.x), "r"(v.y),
                 "r"(v.z), "r"(v.w)
                 : "memory");
}

__device__ __forceinline__ float bf16_lo(uint32_t w) { return __uint_as_float(w << 16); }
__device__ __forceinline__ float bf16_hi(uint32_t w) { return __uint_as_float(w & 0xffff0000u); }

__device__ __forceinline__ float bf16_bits_to_float(uint16_t h) {
    return __uint_as_float(static_cast<uint32_t>(h) << 16);
}

// Two fp32 -> packed bf16x2 (round to nearest even); `lo` lands in the low half.
__device__ __forceinline__ uint32_t pack_bf16x2(float lo, float hi) {
    uint32_t r;
    asm("cvt.rn.bf16x2.f32 %0, %1, %2;" : "=r"(r) : "f"(hi), "f"(lo));
    return r;
}

// ---------------------------------------------------------------------------------------
// 128-point Walsh-Hadamard transform (unnormalised) in the quad layout
// ---------------------------------------------------------------------------------------

// In-register stages over the five in-thread bits of the register index.
__device__ __forceinline__ void fwht_in_thread(float (&v)[kValsPerThread]) {
#pragma unroll
    for (int h = 1; h < kValsPerThread; h <<= 1) {
#pragma unroll
        for (int a = 0; a < kValsPerThread; a += 2 * h) {
#pragma unroll
            for (int b = a; b < a + h; ++b) {
                const float x = v[b], y = v[b + h];
                v[b] = x + y;
                v[b + h] = x - y;
            }
        }
    }
}

// Cross-lane stages over element bits 3 and 4 (lane bits 0 and 1 of the quad).  The lane
// whose bit is 0 keeps x + y, its partner keeps x - y: v' = v * (+-1) + partner.
// Every lane of the warp must call this (full-mask shuffles).
__device__ __forceinline__ void fwht_across_quad(float (&v)[kValsPerThread], int s) {
#pragma unroll
    for (int m = 1; m <= 2; m <<= 1) {
        const float sg = (s & m) ? -1.0f : 1.0f;
#pragma unroll
        for (int j = 0; j < kValsPerThread; ++j) {
            const float p = __shfl_xor_sync(kFullMask, v[j], m);
            v[j] = fmaf(v[j], sg, p);
        }
    }
}

__device__ __forceinline__ void fwht128(float (&v)[kValsPerThread], int s) {
    fwht_in_thread(v);
    fwht_across_quad(v, s);
}

// Sum over the four lanes of a quad (result in every lane).
__device__ __forceinline__ float quad_sum(float x) {
    x += __shfl_xor_sync(kFullMask, x, 1);
    x += __shfl_xor_sync(kFullMask, x, 2);
    return x;
}

// ---------------------------------------------------------------------------------------
// nearest codeword: idx = #{k : r > T_k} for ascending thresholds T_0..T_{L-2}
// (equal to the nearest level with ties to the lower index, T_k = midpoint * scale)
// ---------------------------------------------------------------------------------------

// All-ones when a > b, else zero (a single compare-and-set).
__device__ __forceinline__ uint32_t set_gt(float a, float b) {
    uint32_t d;
    asm("set.gt.u32.f32 %0, %1, %2;" : "=r"(d) : "f"(a), "f"(b));
    return d;
}

template <int L>
__device__ __forceinline__ uint32_t nearest_index(float r, const float (&T)[L - 1]) {
    if constexpr (L == 3) {
        return 0u - (set_gt(r, T[0]) + set_gt(r, T[1]));
    } else if constexpr (L == 4) {
        return 0u - (set_gt(r, T[0]) + set_gt(r, T[1]) + set_gt(r, T[2]));
    } else if constexpr (L == 8) {
        const bool b2 = r > T[3];
        const bool b1 = r > (b2 ? T[5] : T[1]);
        const float t0 = b2 ? (b1 ? T[6] : T[4]) : (b1 ? T[2] : T[0]);
        const bool b0 = r > t0;
        return (b2 ? 4u : 0u) | (b1 ? 2u : 0u) | (b0 ? 1u : 0u);
    } else {
        static_assert(L == 16, "levels must be 3, 4, 8 or 16");
        const bool b3 = r > T[7];
        const bool b2 = r > (b3 ? T[11] : T[3]);
        const float t1 = b3 ? (b2 ? T[13] : T[9]) : (b2 ? T[5] : T[1]);
        const bool b1 = r > t1;
        const float u0 = b1 ? T[2] : T[0], u1 = b1 ? T[6] : T[4];
        const float u2 = b1 ? T[10] : T[8], u3 = b1 ? T[14] : T[12];
        const float t0 = b3 ? (b2 ? u3 : u2) : (b2 ? u1 : u0);
        const bool b0 = r > t0;
        return (b3 ? 8u : 0u) | (b2 ? 4u : 0u) | (b1 ? 2u : 0u) | (b0 ? 1u : 0u);
    }
}

}  // namespace dev
}  // namespace cq
