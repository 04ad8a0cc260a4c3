"""Comparison helpers for GPU-vs-oracle parity (test infrastructure).

Tolerances (the method's floating point leaves these to be fixed; each is derived from
the arithmetic of the fp32 GPU path against the fp64 oracle):
  * indices   bit-exact, except a flip to the ADJACENT index where the oracle's fp64
              component u lies within 1e-5 / sqrt(128) of the midpoint between the two
              codewords (|sqrt(128) (u - m)| <= 1e-5); flips may affect at most
              max(1, 1e-6 * n) of n elements;
  * norms     fp16 bit-exact, except +-1 ulp where the exact group norm lies within 1e-6
              (relative) of the rounding midpoint between the two fp16 values;
  * dequant   fp32 output: relative L2 error <= 1e-5 per group against the oracle's
              dequantisation of the SAME packed input; bf16 output: every element is a
              round-to-nearest bf16 of the oracle value up to 1e-4 of an ulp plus 1e-6 of
              the group's L2 norm (the fp32 transform's own absolute error);
  * GEMV      relative L2 error <= 1e-3 per output vector, SAME packed input.
"""
from __future__ import annotations

import math

import numpy as np

INDEX_BAND = 1e-5
FLIP_FRACTION = 1e-6
NORM_TIE_BAND = 1e-6
DEQ_REL_L2 = 1e-5
GEMV_REL_L2 = 1e-3
BF16_ABS_FROM_NORM = 1e-6


def unpack_fields(packed: np.ndarray, field_bits: int, g: int = 128) -> np.ndarray:
    """LSB-first fields of every group block (numpy.unpackbits, independent of both sides)."""
    p = np.ascontiguousarray(packed, np.uint8)
    blk = g * field_bits // 8
    bits = np.unpackbits(p.reshape(-1, blk), axis=-1, bitorder="little")
    bits = bits.reshape(-1, g, field_bits).astype(np.int64)
    return (bits * (1 << np.arange(field_bits))).sum(-1).reshape(-1, g)


def field_bits(bits: int) -> int:
    return 2 if bits == 0 else bits


def check_indices(gpu_packed, ora_packed, u, bits, codebook, what=""):
    """Assert index parity within the boundary band; returns the number of flips."""
    fb = field_bits(bits)
    gi = unpack_fields(gpu_packed, fb)
    oi = unpack_fields(ora_packed, fb)
    diff = gi != oi
    n = gi.size
    nflip = int(diff.sum())
    if nflip:
        g, o = gi[diff], oi[diff]
        assert np.all(np.abs(g - o) == 1), f"{what}: non-adjacent index flip"
        k = np.minimum(g, o)
        cb = np.asarray(codebook, np.float64)
        mid = (cb[k] + cb[k + 1]) / 2
        uu = np.asarray(u, np.float64).reshape(-1, 128)[diff]
        dist = np.abs(math.sqrt(128) * (uu - mid))
        assert np.all(dist <= INDEX_BAND), f"{what}: flip {dist.max():.3g} outside the band"
        assert nflip <= max(1, int(FLIP_FRACTION * n)), f"{what}: {nflip} flips of {n}"
    return nflip


def check_norms(gpu_norms, ora_norms, exact_norm, what=""):
    """fp16 norms equal, or one ulp apart at a rounding tie (relative band 1e-6)."""
    g = np.asarray(gpu_norms).reshape(-1).view(np.uint16)
    o = np.asarray(ora_norms).reshape(-1).view(np.uint16)
    d = g != o
    if d.any():
        gv = g[d].view(np.float16).astype(np.float64)
        ov = o[d].view(np.float16).astype(np.float64)
        assert np.all(np.abs(g[d].astype(np.int64) - o[d].astype(np.int64)) == 1), \
            f"{what}: norm differs by more than one ulp"
        mid = (gv + ov) / 2
        ex = np.asarray(exact_norm, np.float64).reshape(-1)[d]
        assert np.all(np.abs(ex - mid) <= NORM_TIE_BAND * ex), f"{what}: norm not at a tie"
    return int(d.sum())


def group_norms(w: np.ndarray, cols: int) -> np.ndarray:
    """Exact (fp64) L2 norm of every zero-padded 128-group of w [rows, cols]."""
    w = np.asarray(w, np.float64)
    rows = w.shape[0]
    G = -(-cols // 128)
    pad = np.zeros((rows, G * 128))
    pad[:, :cols] = w
    return np.linalg.norm(pad.reshape(rows, G, 128), axis=-1)


def check_dequant_f32(gpu_out, ora_out, cols, what=""):
    g = np.asarray(gpu_out, np.float64)
    o = np.asarray(ora_out, np.float64)
    rows = g.shape[0]
    G = -(-cols // 128)
    gp = np.zeros((rows, G * 128))
    op = np.zeros((rows, G * 128))
    gp[:, :cols], op[:, :cols] = g, o
    err = np.linalg.norm((gp - op).reshape(rows, G, 128), axis=-1)
    ref = np.linalg.norm(op.reshape(rows, G, 128), axis=-1)
    bad = err > DEQ_REL_L2 * np.maximum(ref, 1e-30)
    bad &= ~((ref == 0) & (err == 0))
    assert not bad.any(), f"{what}: {int(bad.sum())} groups over rel L2 {DEQ_REL_L2}, worst " \
                          f"{float(np.max(err / np.maximum(ref, 1e-30))):.3g}"


def bf16_to_f64(bits_u16: np.ndarray) -> np.ndarray:
    return (np.asarray(bits_u16, np.uint16).astype(np.uint32) << np.uint32(16)).view(np.float32).astype(np.float64)


def check_dequant_bf16(gpu_bits, ora_out, cols, what=""):
    """Each bf16 output is a nearest bf16 of the oracle value, up to the fp32 pipeline's own
    error: |gpu - oracle| <= (0.5 + 1e-4) ulp_bf16 + 1e-6 * ||oracle group||_2.  (The fp32
    transform's absolute error scales with the group norm, not with the element, so a tiny
    element next to a bf16 rounding midpoint may round either way.)"""
    o = np.asarray(ora_out, np.float64)
    rows = o.shape[0] if o.ndim == 2 else 1
    o = o.reshape(rows, cols)
    g = bf16_to_f64(gpu_bits).reshape(rows, cols)
    G = -(-cols // 128)
    op = np.zeros((rows, G * 128))
    op[:, :cols] = o
    gn = np.repeat(np.linalg.norm(op.reshape(rows, G, 128), axis=-1), 128, axis=1)[:, :cols]
    mag = np.maximum(np.abs(o), np.abs(g))
    ulp = np.where(mag > 0, np.exp2(np.floor(np.log2(np.maximum(mag, 1e-38))) - 7), 0.0)
    err = np.abs(g - o)
    bad = err > (0.5 + 1e-4) * ulp + BF16_ABS_FROM_NORM * gn + 1e-38
    assert not bad.any(), f"{what}: {int(bad.sum())} bf16 outputs are not nearest"


def check_gemv(gpu_y, ora_y, what=""):
    g = np.asarray(gpu_y, np.float64)
    o = np.asarray(ora_y, np.float64)
    for b in range(o.shape[0]):
        rel = np.linalg.norm(g[b] - o[b]) / max(np.linalg.norm(o[b]), 1e-30)
        assert rel <= GEMV_REL_L2, f"{what}: batch row {b} rel L2 {rel:.3g}"
    return float(max(np.linalg.norm(g[b] - o[b]) / max(np.linalg.norm(o[b]), 1e-30)
                     for b in range(o.shape[0])))


# ------------------------------------------------------------------------------------------
# guard bytes around output buffers (stands in for a memory checker: a kernel that writes past
# either end of its output changes the margins)
# ------------------------------------------------------------------------------------------

GUARD_BYTES = 4096
GUARD_FILL = 0xA5


def guarded_empty(shape, dtype, device):
    """(base, t): `t` of `shape` and `dtype` lies inside `base`, a 1-D allocation with
    GUARD_BYTES of GUARD_FILL before and after it.  t starts GUARD_BYTES into base, so it keeps
    base's 16-byte alignment."""
    import torch
    numel = 1
    for d in shape:
        numel *= int(d)
    esz = torch.empty((), dtype=dtype).element_size()
    g = GUARD_BYTES // esz
    base = torch.empty(numel + 2 * g, dtype=dtype, device=device)
    base.view(torch.uint8).fill_(GUARD_FILL)
    return base, base[g:g + numel].view(tuple(shape))


def guard_intact(base, t) -> bool:
    """True when both margins of `base` around `t` still hold GUARD_FILL."""
    import torch
    b = base.view(torch.uint8)
    n = t.numel() * t.element_size()
    return bool((b[:GUARD_BYTES] == GUARD_FILL).all() and (b[GUARD_BYTES + n:] == GUARD_FILL).all())
