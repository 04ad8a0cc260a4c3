"""CPU oracle for CQ quantisation (TEST INFRASTRUCTURE ONLY).

Thin ctypes wrapper over ``cq_oracle.c``: a plain fp64 implementation of Cactus-Quants
group-wise Hadamard/codebook quantisation written from the method's description (pages
"Cactus Quants CQ2-bit Quantization", "How CQ2-bit Quantization Contributes to Needle 2's
Small Footprint", "How Quantization Codebooks Are Trained in Cactus Quants").

Only the test suite, ``__graft_entry__.smoke()`` and the CPU-baseline leg of ``bench.py``
may import this package.  The product library (``hadamard_codebook_bit_b200``) never
imports it and shares no code with it.

Parity status: every exported function is pinned by ``tests/test_oracle_pins.py``
against closed forms, NumPy/SciPy library routines or values printed on the pages.
"""
from __future__ import annotations

import ctypes
import functools
import os
import subprocess

import numpy as np

_HERE = os.path.dirname(os.path.abspath(__file__))
_SRC = os.path.join(_HERE, "cq_oracle.c")
_HDR = os.path.join(_HERE, "cq_oracle.h")
_LIB = os.path.join(_HERE, "libcq_oracle.so")

F32, BF16, F64 = 0, 1, 2
TERNARY = 0

_lib = None


def build(force: bool = False) -> str:
    """Compile the oracle with gcc (plain C11, fp64, no FMA contraction)."""
    stale = (not os.path.exists(_LIB)) or any(
        os.path.getmtime(p) > os.path.getmtime(_LIB) for p in (_SRC, _HDR))
    if force or stale:
        tmp = _LIB + f".tmp{os.getpid()}"
        subprocess.check_call([
            "gcc", "-std=c11", "-O2", "-ffp-contract=off", "-fno-fast-math", "-fPIC",
            "-shared", "-pthread", "-o", tmp, _SRC, "-lm"])
        os.replace(tmp, _LIB)
    return _LIB


def lib() -> ctypes.CDLL:
    global _lib
    if _lib is None:
        build()
        L = ctypes.CDLL(_LIB)
        P = ctypes.c_void_p
        i64, i32, u32, sz = ctypes.c_int64, ctypes.c_int, ctypes.c_uint32, ctypes.c_size_t
        L.cqo_hadamard.argtypes = [i32, P]
        L.cqo_mt_uint32.argtypes = [u32, sz, P]
        L.cqo_randn.argtypes = [u32, sz, P]
        L.cqo_lloyd_max.argtypes = [i32, i32, i32, u32, P]
        L.cqo_lloyd_on_sorted.argtypes = [P, i32, i32, i32, P]
        L.cqo_codebook.argtypes = [i32, i32, u32, P]
        L.cqo_levels.argtypes = [i32]
        L.cqo_field_bits.argtypes = [i32]
        L.cqo_packed_bytes.argtypes = [i64, i64, i32, i32]
        L.cqo_packed_bytes.restype = sz
        L.cqo_norm_bytes.argtypes = [i64, i64, i32]
        L.cqo_norm_bytes.restype = sz
        L.cqo_f64_to_f16.argtypes = [ctypes.c_double]
        L.cqo_f64_to_f16.restype = ctypes.c_uint16
        L.cqo_f16_to_f64.argtypes = [ctypes.c_uint16]
        L.cqo_f16_to_f64.restype = ctypes.c_double
        L.cqo_f64_to_bf16.argtypes = [ctypes.c_double]
        L.cqo_f64_to_bf16.restype = ctypes.c_uint16
        L.cqo_quantize.argtypes = [P, i32, i64, i64, i32, i32, P, P, P, P, i32]
        L.cqo_dequantize.argtypes = [P, P, i64, i64, i32, i32, P, P, i32]
        L.cqo_dequant_gemv.argtypes = [P, P, i64, i64, i32, i32, P, P, i32, i32, P, i32]
        L.cqo_unpack_index.argtypes = [P, i32, i32]
        L.cqo_rel_mse.argtypes = [P, i32, P, i64]
        L.cqo_rel_mse.restype = ctypes.c_double
        _lib = L
    return _lib


def _ptr(a: np.ndarray):
    assert a.flags["C_CONTIGUOUS"]
    return a.ctypes.data_as(ctypes.c_void_p)


def _dtype_code(a: np.ndarray) -> int:
    if a.dtype == np.float32:
        return F32
    if a.dtype == np.float64:
        return F64
    if a.dtype == np.uint16:  # bf16 bit patterns
        return BF16
    raise TypeError(f"oracle takes float32, float64 or bf16 bits as uint16, not {a.dtype}")


def default_threads() -> int:
    return lib().cqo_default_threads()


def hadamard(g: int) -> np.ndarray:
    H = np.empty((g, g), np.float64)
    if lib().cqo_hadamard(g, _ptr(H)) != 0:
        raise ValueError("group size must be a power of two")
    return H


def mt_uint32(seed: int, n: int) -> np.ndarray:
    out = np.empty(n, np.uint32)
    lib().cqo_mt_uint32(seed, n, _ptr(out))
    return out


def randn(seed: int, n: int) -> np.ndarray:
    out = np.empty(n, np.float64)
    lib().cqo_randn(seed, n, _ptr(out))
    return out


def lloyd_max(levels: int, samples: int = 400000, iters: int = 200, seed: int = 0) -> np.ndarray:
    out = np.empty(levels, np.float64)
    if lib().cqo_lloyd_max(levels, samples, iters, seed, _ptr(out)) != 0:
        raise ValueError("bad Lloyd-Max arguments")
    return out


def lloyd_on_sorted(x: np.ndarray, levels: int, iters: int) -> np.ndarray:
    x = np.ascontiguousarray(np.sort(np.asarray(x, np.float64)))
    out = np.empty(levels, np.float64)
    if lib().cqo_lloyd_on_sorted(_ptr(x), x.size, levels, iters, _ptr(out)) != 0:
        raise ValueError("bad Lloyd arguments")
    return out


def levels(bits: int) -> int:
    return lib().cqo_levels(bits)


def field_bits(bits: int) -> int:
    return lib().cqo_field_bits(bits)


@functools.lru_cache(maxsize=None)
def _codebook_cached(bits: int, group_size: int, seed: int) -> np.ndarray:
    out = np.zeros(16, np.float32)
    n = lib().cqo_codebook(bits, group_size, seed, _ptr(out))
    if n < 0:
        raise ValueError("bad codebook arguments")
    out = out[:n].copy()
    out.flags.writeable = False
    return out


def codebook(bits: int, group_size: int = 128, seed: int = 0) -> np.ndarray:
    """Codebook (fp32, ascending), cached per arguments like the pages' lru_cache."""
    return _codebook_cached(int(bits), int(group_size), int(seed)).copy()


def packed_bytes(rows: int, cols: int, bits: int, group_size: int = 128) -> int:
    return int(lib().cqo_packed_bytes(rows, cols, bits, group_size))


def norm_bytes(rows: int, cols: int, group_size: int = 128) -> int:
    return int(lib().cqo_norm_bytes(rows, cols, group_size))


def f64_to_f16_bits(x: float) -> int:
    return int(lib().cqo_f64_to_f16(float(x)))


def f16_bits_to_f64(h: int) -> float:
    return float(lib().cqo_f16_to_f64(int(h)))


def f64_to_bf16_bits(x: float) -> int:
    return int(lib().cqo_f64_to_bf16(float(x)))


def quantize(w: np.ndarray, bits: int, group_size: int = 128, codebook_: np.ndarray | None = None,
             want_u: bool = False, nthreads: int = 0):
    """Return (packed uint8 [rows, G, g*b/8], norms uint16 fp16 bits [rows, G][, u fp64])."""
    w = np.ascontiguousarray(w)
    if w.ndim != 2:
        raise ValueError("w must be 2-D [rows, cols]")
    rows, cols = w.shape
    cb = np.ascontiguousarray(codebook(bits, group_size) if codebook_ is None else codebook_,
                              dtype=np.float32)
    G = -(-cols // group_size)
    blk = group_size * field_bits(bits) // 8
    packed = np.zeros((rows, G, blk), np.uint8)
    norms = np.zeros((rows, G), np.uint16)
    u = np.zeros((rows, G, group_size), np.float64) if want_u else None
    rc = lib().cqo_quantize(_ptr(w), _dtype_code(w), rows, cols, bits, group_size, _ptr(cb),
                            _ptr(packed), _ptr(norms), _ptr(u) if want_u else None, nthreads)
    if rc != 0:
        raise ValueError("bad quantize arguments")
    return (packed, norms, u) if want_u else (packed, norms)


def dequantize(packed: np.ndarray, norms: np.ndarray, rows: int, cols: int, bits: int,
               group_size: int = 128, codebook_: np.ndarray | None = None,
               nthreads: int = 0) -> np.ndarray:
    cb = np.ascontiguousarray(codebook(bits, group_size) if codebook_ is None else codebook_,
                              dtype=np.float32)
    packed = np.ascontiguousarray(packed, np.uint8)
    norms = np.ascontiguousarray(norms, np.uint16)
    out = np.empty((rows, cols), np.float64)
    rc = lib().cqo_dequantize(_ptr(packed), _ptr(norms), rows, cols, bits, group_size, _ptr(cb),
                              _ptr(out), nthreads)
    if rc != 0:
        raise ValueError("bad dequantize arguments")
    return out


def fake_quantize(w: np.ndarray, bits: int, group_size: int = 128,
                  codebook_: np.ndarray | None = None, nthreads: int = 0) -> np.ndarray:
    """W_hat [rows, cols] fp64 = dequantize(quantize(w)): the de-quantised tensor the pages'
    cq_quantize returns (page "Cactus Quants CQ2-bit Quantization", "The CQ2-bit
    Implementation Pipeline", steps 1-6).  The inverse rotation scales by the stored fp16
    norm, so the result is what a deployment reconstructs from the stored form."""
    w = np.ascontiguousarray(w)
    rows, cols = w.shape
    packed, norms = quantize(w, bits, group_size, codebook_, nthreads=nthreads)
    return dequantize(packed, norms, rows, cols, bits, group_size, codebook_, nthreads)


def dequant_gemv(packed: np.ndarray, norms: np.ndarray, rows: int, cols: int, bits: int,
                 x: np.ndarray, group_size: int = 128, codebook_: np.ndarray | None = None,
                 nthreads: int = 0) -> np.ndarray:
    """y [batch, rows] = W_hat x for x [batch, cols] (float32/float64 or bf16 bits)."""
    cb = np.ascontiguousarray(codebook(bits, group_size) if codebook_ is None else codebook_,
                              dtype=np.float32)
    x = np.ascontiguousarray(x)
    if x.ndim == 1:
        x = x[None, :]
    batch = x.shape[0]
    packed = np.ascontiguousarray(packed, np.uint8)
    norms = np.ascontiguousarray(norms, np.uint16)
    y = np.empty((batch, rows), np.float64)
    rc = lib().cqo_dequant_gemv(_ptr(packed), _ptr(norms), rows, cols, bits, group_size, _ptr(cb),
                                _ptr(x), _dtype_code(x), batch, _ptr(y), nthreads)
    if rc != 0:
        raise ValueError("bad gemv arguments")
    return y


def unpack_index(block: np.ndarray, bits: int, i: int) -> int:
    block = np.ascontiguousarray(block, np.uint8)
    return int(lib().cqo_unpack_index(_ptr(block), field_bits(bits), i))


def rel_mse(w: np.ndarray, w_hat: np.ndarray) -> float:
    w = np.ascontiguousarray(w)
    w_hat = np.ascontiguousarray(w_hat, np.float64)
    return float(lib().cqo_rel_mse(_ptr(w), _dtype_code(w), _ptr(w_hat), w.size))
