// cq_synth.cu -- seeded synthetic inputs on the GPU (test and benchmark infrastructure).
//
// Holds no quantisation arithmetic: only a counter-based normal generator, defined so the
// NumPy implementation in synth/__init__.py produces the same bits:
//   * Philox4x32-10 (Salmon, Moraes, Dror, Shaw, "Parallel random numbers: as easy as
//     1, 2, 3", SC'11): key (seed, tensor_id), counter (m_lo, m_hi, 0, 0) for pair m;
//   * Box-Muller on two 53-bit uniforms, u1 in (0, 1], u2 in [0, 1);
//   * log, sin and cos evaluated by fixed polynomials with plain IEEE operations in a fixed
//     order (this file is compiled with -fmad=false, so no fused multiply-add);
//   * element 2m is rho*cos(theta), element 2m+1 is rho*sin(theta); value = sigma * z,
//     rounded to fp32, then (for bf16) to bf16, both round to nearest even.
#include <cstdint>

#include <cuda_runtime.h>

namespace {

__device__ __forceinline__ void philox_round(uint32_t& c0, uint32_t& c1, uint32_t& c2,
                                             uint32_t& c3, uint32_t k0, uint32_t k1) {
    const uint32_t lo0 = 0xD2511F53u * c0, hi0 = __umulhi(0xD2511F53u, c0);
    const uint32_t lo1 = 0xCD9E8D57u * c2, hi1 = __umulhi(0xCD9E8D57u, c2);
    const uint32_t n0 = hi1 ^ c1 ^ k0, n2 = hi0 ^ c3 ^ k1;
    c0 = n0;
    c1 = lo1;
    c2 = n2;
    c3 = lo0;
}

__device__ __forceinline__ uint4 philox4x32_10(uint32_t c0, uint32_t c1, uint32_t k0, uint32_t k1) {
    uint32_t c2 = 0, c3 = 0;
#pragma unroll
    for (int r = 0; r < 10; ++r) {
        philox_round(c0, c1, c2, c3, k0, k1);
        k0 += 0x9E3779B9u;
        k1 += 0xBB67AE85u;
    }
    return make_uint4(c0, c1, c2, c3);
}

__device__ double poly_log(double u) {
    int e;
    double m = frexp(u, &e);  // u = m * 2^e, m in [0.5, 1)
    if (m < 0.7071067811865476) {
        m = m * 2.0;
        e = e - 1;
    }
    const double s = (m - 1.0) / (m + 1.0);
    const double z = s * s;
    double p = 0.043478260869565216;
    p = p * z + 0.047619047619047616;
    p = p * z + 0.05263157894736842;
    p = p * z + 0.058823529411764705;
    p = p * z + 0.06666666666666667;
    p = p * z + 0.07692307692307693;
    p = p * z + 0.09090909090909091;
    p = p * z + 0.1111111111111111;
    p = p * z + 0.14285714285714285;
    p = p * z + 0.2;
    p = p * z + 0.3333333333333333;
    p = p * z + 1.0;
    return static_cast<double>(e) * 0.6931471805599453 + 2.0 * s * p;
}

__device__ void poly_sincos_quarter(double x, double* s_out, double* c_out) {
    const double z = x * x;
    double s = -3.868170170630684e-23;
    s = s * z + 1.9572941063391263e-20;
    s = s * z + -8.22063524662433e-18;
    s = s * z + 2.8114572543455206e-15;
    s = s * z + -7.647163731819816e-13;
    s = s * z + 1.6059043836821613e-10;
    s = s * z + -2.505210838544172e-08;
    s = s * z + 2.7557319223985893e-06;
    s = s * z + -0.0001984126984126984;
    s = s * z + 0.008333333333333333;
    s = s * z + -0.16666666666666666;
    s = s * z + 1.0;
    double c = 1.6117375710961184e-24;
    c = c * z + -8.896791392450574e-22;
    c = c * z + 4.110317623312165e-19;
    c = c * z + -1.5619206968586225e-16;
    c = c * z + 4.779477332387385e-14;
    c = c * z + -1.1470745597729725e-11;
    c = c * z + 2.08767569878681e-09;
    c = c * z + -2.755731922398589e-07;
    c = c * z + 2.48015873015873e-05;
    c = c * z + -0.001388888888888889;
    c = c * z + 0.041666666666666664;
    c = c * z + -0.5;
    c = c * z + 1.0;
    *s_out = x * s;
    *c_out = c;
}

__device__ __forceinline__ uint16_t f32_to_bf16_rne(float f) {
    const uint32_t u = __float_as_uint(f);
    if ((u & 0x7f800000u) == 0x7f800000u) return static_cast<uint16_t>((u >> 16) | ((u & 0xffffu) ? 0x40u : 0u));
    return static_cast<uint16_t>((u + 0x7fffu + ((u >> 16) & 1u)) >> 16);
}

// out: n elements starting at element index `offset` of stream (seed, tensor_id).
__global__ void fill_normal_kernel(void* out, int is_bf16, long long n, long long offset,
                                   uint32_t seed, uint32_t tensor_id, double sigma) {
    const long long first_pair = offset >> 1;
    const long long last_pair = (offset + n - 1) >> 1;
    const long long npairs = last_pair - first_pair + 1;
    for (long long t = blockIdx.x * static_cast<long long>(blockDim.x) + threadIdx.x; t < npairs;
         t += static_cast<long long>(gridDim.x) * blockDim.x) {
        const unsigned long long m = static_cast<unsigned long long>(first_pair + t);
        const uint4 x = philox4x32_10(static_cast<uint32_t>(m), static_cast<uint32_t>(m >> 32),
                                      seed, tensor_id);
        const double u1 = ((static_cast<double>(x.x >> 5) * 67108864.0 +
                            static_cast<double>(x.y >> 6)) + 1.0) * 1.1102230246251565e-16;
        const double u2 = (static_cast<double>(x.z >> 5) * 67108864.0 +
                           static_cast<double>(x.w >> 6)) * 1.1102230246251565e-16;
        const double rho = sqrt(-2.0 * poly_log(u1));
        const double t4 = u2 * 4.0;
        const double qd = floor(t4);
        const double f = t4 - qd;
        double S, C;
        poly_sincos_quarter(f * 1.5707963267948966, &S, &C);
        const int qi = static_cast<int>(qd);
        const double cth = qi == 0 ? C : qi == 1 ? -S : qi == 2 ? -C : S;
        const double sth = qi == 0 ? S : qi == 1 ? C : qi == 2 ? -S : -C;
        const double z[2] = {rho * cth, rho * sth};
#pragma unroll
        for (int h = 0; h < 2; ++h) {
            const long long e = 2 * static_cast<long long>(m) + h - offset;
            if (e < 0 || e >= n) continue;
            const float v = static_cast<float>(sigma * z[h]);
            if (is_bf16)
                static_cast<uint16_t*>(out)[e] = f32_to_bf16_rne(v);
            else
                static_cast<float*>(out)[e] = v;
        }
    }
}

}  // namespace

extern "C" int cqs_fill_normal(void* out, int is_bf16, long long n, long long offset,
                               unsigned int seed, unsigned int tensor_id, double sigma,
                               void* stream) {
    if (!out || n <= 0 || offset < 0) return 1;
    const long long npairs = ((offset + n - 1) >> 1) - (offset >> 1) + 1;
    long long blocks = (npairs + 255) / 256;
    if (blocks > 148LL * 16) blocks = 148LL * 16;
    fill_normal_kernel<<<static_cast<int>(blocks), 256, 0, static_cast<cudaStream_t>(stream)>>>(
        out, is_bf16, n, offset, seed, tensor_id, sigma);
    return cudaGetLastError() == cudaSuccess ? 0 : 3;
}
