"""Seeded synthetic inputs for tests and the benchmark (no quantisation arithmetic here).

Generator ("Philox/Box-Muller normal stream"), identical on the host (NumPy, this file)
and on the GPU (``cq_synth.cu``, compiled without fused multiply-add):

* Philox4x32-10 (Salmon et al., SC'11) with key ``(seed, tensor_id)`` and counter
  ``(m & 0xffffffff, m >> 32, 0, 0)`` for element pair ``m``;
* two 53-bit uniforms ``u1 = (((x0>>5)*2^26 + (x1>>6)) + 1) * 2^-53`` in (0, 1] and
  ``u2 = ((x2>>5)*2^26 + (x3>>6)) * 2^-53`` in [0, 1);
* ``rho = sqrt(-2 ln u1)``, ``theta = 2 pi u2``; log / sin / cos by fixed polynomials;
* element ``2m`` is ``rho cos(theta)``, element ``2m + 1`` is ``rho sin(theta)``;
* the stored value is ``sigma * z`` rounded to fp32 and then, for bf16, to bf16 (both
  round to nearest even).

Any element of any tensor can therefore be regenerated on the host for sampled checks.
"""
from __future__ import annotations

import ctypes
import os
import shutil
import subprocess

import numpy as np

_HERE = os.path.dirname(os.path.abspath(__file__))
_CU = os.path.join(_HERE, "cq_synth.cu")
_LIB = os.path.join(_HERE, "libcq_synth.so")

_M0, _M1 = np.uint64(0xD2511F53), np.uint64(0xCD9E8D57)
_W0, _W1 = 0x9E3779B9, 0xBB67AE85
_MASK32 = np.uint64(0xFFFFFFFF)
_TWO_M53 = 1.1102230246251565e-16

_INV_ODD = [1.0, 0.3333333333333333, 0.2, 0.14285714285714285, 0.1111111111111111,
            0.09090909090909091, 0.07692307692307693, 0.06666666666666667,
            0.058823529411764705, 0.05263157894736842, 0.047619047619047616,
            0.043478260869565216]
_SIN = [1.0, -0.16666666666666666, 0.008333333333333333, -0.0001984126984126984,
        2.7557319223985893e-06, -2.505210838544172e-08, 1.6059043836821613e-10,
        -7.647163731819816e-13, 2.8114572543455206e-15, -8.22063524662433e-18,
        1.9572941063391263e-20, -3.868170170630684e-23]
_COS = [1.0, -0.5, 0.041666666666666664, -0.001388888888888889, 2.48015873015873e-05,
        -2.755731922398589e-07, 2.08767569878681e-09, -1.1470745597729725e-11,
        4.779477332387385e-14, -1.5619206968586225e-16, 4.110317623312165e-19,
        -8.896791392450574e-22, 1.6117375710961184e-24]


# ------------------------------------------------------------------------------------------
# host implementation
# ------------------------------------------------------------------------------------------

def philox4x32_10(m: np.ndarray, seed: int, tensor_id: int):
    """Philox4x32-10 on counters (m_lo, m_hi, 0, 0); returns four uint32 arrays."""
    m = np.asarray(m, np.uint64)
    c0 = m & _MASK32
    c1 = m >> np.uint64(32)
    c2 = np.zeros_like(c0)
    c3 = np.zeros_like(c0)
    k0, k1 = seed & 0xFFFFFFFF, tensor_id & 0xFFFFFFFF
    for _ in range(10):
        p0 = _M0 * c0
        p1 = _M1 * c2
        hi0, lo0 = p0 >> np.uint64(32), p0 & _MASK32
        hi1, lo1 = p1 >> np.uint64(32), p1 & _MASK32
        c0, c1, c2, c3 = hi1 ^ c1 ^ np.uint64(k0), lo1, hi0 ^ c3 ^ np.uint64(k1), lo0
        k0 = (k0 + _W0) & 0xFFFFFFFF
        k1 = (k1 + _W1) & 0xFFFFFFFF
    return c0, c1, c2, c3


def _poly_log(u: np.ndarray) -> np.ndarray:
    m, e = np.frexp(u)
    small = m < 0.7071067811865476
    m = np.where(small, m * 2.0, m)
    e = np.where(small, e - 1, e)
    s = (m - 1.0) / (m + 1.0)
    z = s * s
    p = np.full_like(z, _INV_ODD[-1])
    for c in reversed(_INV_ODD[:-1]):
        p = p * z + c
    return e.astype(np.float64) * 0.6931471805599453 + (2.0 * s) * p


def _poly_sincos(x: np.ndarray):
    z = x * x
    s = np.full_like(z, _SIN[-1])
    for c in reversed(_SIN[:-1]):
        s = s * z + c
    c_ = np.full_like(z, _COS[-1])
    for c in reversed(_COS[:-1]):
        c_ = c_ * z + c
    return x * s, c_


def _normal_pairs(m: np.ndarray, seed: int, tensor_id: int):
    x0, x1, x2, x3 = philox4x32_10(m, seed, tensor_id)
    u1 = (((x0 >> np.uint64(5)).astype(np.float64) * 67108864.0 +
           (x1 >> np.uint64(6)).astype(np.float64)) + 1.0) * _TWO_M53
    u2 = ((x2 >> np.uint64(5)).astype(np.float64) * 67108864.0 +
          (x3 >> np.uint64(6)).astype(np.float64)) * _TWO_M53
    rho = np.sqrt(-2.0 * _poly_log(u1))
    t4 = u2 * 4.0
    qd = np.floor(t4)
    S, C = _poly_sincos((t4 - qd) * 1.5707963267948966)
    q = qd.astype(np.int64)
    cth = np.select([q == 0, q == 1, q == 2], [C, -S, -C], S)
    sth = np.select([q == 0, q == 1, q == 2], [S, C, -S], -C)
    return rho * cth, rho * sth


def normal_f64(n: int, seed: int, tensor_id: int, offset: int = 0) -> np.ndarray:
    """Standard normal deviates (fp64, before scaling) of elements offset..offset+n-1."""
    out = np.empty(n, np.float64)
    chunk = 1 << 22
    for a in range(0, n, chunk):
        b = min(n, a + chunk)
        e0, e1 = offset + a, offset + b - 1
        m = np.arange(e0 >> 1, (e1 >> 1) + 1, dtype=np.uint64)
        z0, z1 = _normal_pairs(m, seed, tensor_id)
        inter = np.empty(2 * m.size, np.float64)
        inter[0::2], inter[1::2] = z0, z1
        out[a:b] = inter[e0 - 2 * (e0 >> 1): e0 - 2 * (e0 >> 1) + (b - a)]
    return out


def f32_to_bf16_bits(x: np.ndarray) -> np.ndarray:
    """fp32 -> bf16 bit patterns, round to nearest even (finite inputs)."""
    u = np.ascontiguousarray(x, np.float32).view(np.uint32).astype(np.uint64)
    return ((u + np.uint64(0x7FFF) + ((u >> np.uint64(16)) & np.uint64(1))) >> np.uint64(16)).astype(np.uint16)


def bf16_bits_to_f32(b: np.ndarray) -> np.ndarray:
    return (np.asarray(b, np.uint16).astype(np.uint32) << np.uint32(16)).view(np.float32)


def normal_host(shape, seed: int, tensor_id: int, sigma: float, dtype: str = "f32",
                offset: int = 0) -> np.ndarray:
    """sigma * N(0,1) of the stream, as float32 or bf16 bits (uint16)."""
    n = int(np.prod(shape))
    v = (sigma * normal_f64(n, seed, tensor_id, offset)).astype(np.float32)
    if dtype == "bf16":
        return f32_to_bf16_bits(v).reshape(shape)
    return v.reshape(shape)


def philox_words(n: int, seed: int, tensor_id: int) -> np.ndarray:
    """First output word x0 of counters 0..n-1 (used for index draws)."""
    return philox4x32_10(np.arange(n, dtype=np.uint64), seed, tensor_id)[0].astype(np.uint64)


# ------------------------------------------------------------------------------------------
# device implementation (libcq_synth.so)
# ------------------------------------------------------------------------------------------

def build(force: bool = False) -> str:
    if force or not os.path.exists(_LIB) or os.path.getmtime(_CU) > os.path.getmtime(_LIB):
        nvcc = "/usr/local/cuda/bin/nvcc" if os.path.exists("/usr/local/cuda/bin/nvcc") else shutil.which("nvcc")
        tmp = _LIB + f".tmp{os.getpid()}"
        subprocess.check_call([nvcc, "-gencode", "arch=compute_100a,code=sm_100a", "-O3",
                               "-fmad=false", "-lineinfo", "-Xcompiler", "-fPIC", "-shared",
                               "-o", tmp, _CU])
        os.replace(tmp, _LIB)
    return _LIB


_dlib = None


def _device_lib():
    global _dlib
    if _dlib is None:
        build()
        L = ctypes.CDLL(_LIB)
        L.cqs_fill_normal.argtypes = [ctypes.c_void_p, ctypes.c_int, ctypes.c_longlong,
                                      ctypes.c_longlong, ctypes.c_uint, ctypes.c_uint,
                                      ctypes.c_double, ctypes.c_void_p]
        _dlib = L
    return _dlib


def fill_normal_(t, seed: int, tensor_id: int, sigma: float, offset: int = 0):
    """Fill a contiguous CUDA tensor (float32 or bfloat16) with the stream, in place."""
    import torch
    if not (t.is_cuda and t.is_contiguous()) or t.dtype not in (torch.float32, torch.bfloat16):
        raise ValueError("need a contiguous float32/bfloat16 CUDA tensor")
    with torch.cuda.device(t.device):
        rc = _device_lib().cqs_fill_normal(t.data_ptr(), int(t.dtype == torch.bfloat16), t.numel(),
                                           offset, seed, tensor_id, sigma,
                                           torch.cuda.current_stream(t.device).cuda_stream)
    if rc != 0:
        raise RuntimeError(f"cqs_fill_normal failed ({rc})")
    return t
