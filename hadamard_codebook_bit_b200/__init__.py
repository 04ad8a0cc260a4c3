"""Python binding of libcq: CQ (Cactus-Quants) Hadamard/codebook weight quantisation on B200.

The functions below only marshal arguments to the C ABI declared in ``include/cq.h``;
every step of quantise / dequantise / dequant-GEMV runs in the CUDA kernels of
``libcq.so``.  PyTorch supplies device memory and the current CUDA stream.  There is no
CPU fallback: if ``libcq.so`` is missing or a call fails, an exception is raised.

Layout (page "How CQ2-bit Quantization Contributes to Needle 2's Small Footprint",
"Per-Group Storage Breakdown"): ``packed`` is uint8 ``[rows, G, 16*b]`` (b = 2 for
ternary), ``norms`` is float16 ``[rows, G]`` with ``G = ceil(cols / 128)``.
"""
from __future__ import annotations

import ctypes
import os

import numpy as np

_HERE = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(_HERE, "libcq.so")

TERNARY = 0
GROUP_SIZE = 128
CQ_F32, CQ_BF16 = 0, 1

_STATUS = {0: "CQ_OK", 1: "CQ_ERR_INVALID_ARG", 2: "CQ_ERR_UNSUPPORTED", 3: "CQ_ERR_CUDA",
           4: "CQ_ERR_ALIGNMENT", 5: "CQ_ERR_WORKSPACE"}

# Every symbol include/cq.h declares (checked by the CPU test suite).
EXPORTS = ("cq_status_string", "cq_version", "cq_device_status", "cq_codebook", "cq_packed_bytes",
           "cq_norm_bytes", "cq_quantize", "cq_dequantize", "cq_dequant_gemv",
           "cq_gemv_workspace_bytes", "cq_dequant_gemv_static", "cq_quantize_batch",
           "cq_dequantize_batch", "cq_dequant_gemv_batch", "cq_fake_quantize", "cq_fake_quantize_batch")


class CQError(RuntimeError):
    def __init__(self, status: int, what: str):
        self.status = status
        super().__init__(f"{what}: {lib().cq_status_string(status).decode()}")


_lib = None


def lib() -> ctypes.CDLL:
    """Load libcq.so (raises if it has not been built)."""
    global _lib
    if _lib is None:
        if not os.path.exists(LIB_PATH):
            raise ImportError(f"libcq.so not built at {LIB_PATH}; run "
                              "`python -m hadamard_codebook_bit_b200.build`")
        L = ctypes.CDLL(LIB_PATH)
        P, ll, i, sz = ctypes.c_void_p, ctypes.c_longlong, ctypes.c_int, ctypes.c_size_t
        L.cq_status_string.argtypes = [i]
        L.cq_status_string.restype = ctypes.c_char_p
        L.cq_version.restype = i
        L.cq_device_status.argtypes = [i, P]
        L.cq_codebook.argtypes = [i, i, ctypes.c_ulonglong, P, P]
        L.cq_packed_bytes.argtypes = [ll, ll, i, i]
        L.cq_packed_bytes.restype = sz
        L.cq_norm_bytes.argtypes = [ll, ll, i]
        L.cq_norm_bytes.restype = sz
        L.cq_quantize.argtypes = [P, i, ll, ll, i, i, P, P, P, P]
        L.cq_dequantize.argtypes = [P, P, ll, ll, i, i, P, P, i, P]
        L.cq_dequant_gemv.argtypes = [P, P, ll, ll, i, i, P, P, i, P, P, sz, P]
        L.cq_gemv_workspace_bytes.argtypes = [ll, i]
        L.cq_gemv_workspace_bytes.restype = sz
        L.cq_dequant_gemv_static.argtypes = [P, P, ll, ll, i, i, P, P, i, P, P]
        L.cq_quantize_batch.argtypes = [P, i, i, i, i, P, P]
        L.cq_dequantize_batch.argtypes = [P, i, i, i, P, i, P]
        L.cq_dequant_gemv_batch.argtypes = [P, i, i, i, P, P]
        L.cq_fake_quantize.argtypes = [P, i, ll, ll, i, i, P, P, P, P, i, P]
        L.cq_fake_quantize_batch.argtypes = [P, i, i, i, i, P, i, P]
        _lib = L
    return _lib


def _check(rc: int, what: str) -> None:
    if rc != 0:
        raise CQError(rc, what)


def device_status(reset: bool = False) -> int:
    """Watchdog word of the current device (0 = no kernel wait ever gave up); synchronises."""
    v = ctypes.c_uint(0)
    _check(lib().cq_device_status(int(reset), ctypes.byref(v)), "cq_device_status")
    return int(v.value)


def field_bits(bits: int) -> int:
    return 2 if bits == TERNARY else bits


def levels(bits: int) -> int:
    return 3 if bits == TERNARY else 1 << bits


def codebook(bits: int, group_size: int = GROUP_SIZE, seed: int = 0) -> np.ndarray:
    """Default Lloyd-Max / ternary codebook, fp32 ascending (host routine, memoised)."""
    out = np.zeros(16, np.float32)
    n = ctypes.c_int(0)
    _check(lib().cq_codebook(bits, group_size, seed, out.ctypes.data_as(ctypes.c_void_p),
                             ctypes.byref(n)), "cq_codebook")
    return out[:n.value].copy()


def packed_bytes(rows: int, cols: int, bits: int, group_size: int = GROUP_SIZE) -> int:
    return int(lib().cq_packed_bytes(rows, cols, bits, group_size))


def norm_bytes(rows: int, cols: int, group_size: int = GROUP_SIZE) -> int:
    return int(lib().cq_norm_bytes(rows, cols, group_size))


def gemv_workspace_bytes(cols: int, batch: int) -> int:
    return int(lib().cq_gemv_workspace_bytes(cols, batch))


# ------------------------------------------------------------------------------------------
# torch-facing wrappers (device tensors, current stream)
# ------------------------------------------------------------------------------------------

def _torch():
    import torch
    return torch


def _stream(device) -> int:
    torch = _torch()
    return torch.cuda.current_stream(device).cuda_stream


def _dev_ptr(t, name: str) -> int:
    if not t.is_cuda:
        raise ValueError(f"{name} must be a CUDA tensor")
    if not t.is_contiguous():
        raise ValueError(f"{name} must be contiguous")
    return t.data_ptr()


# The C ABI takes plain pointers and sizes, so a buffer smaller than a call touches would make
# the kernels read or write past its end.  The binding checks every buffer first (dtype and
# byte count: _fits, _check_stored, _check_x), then takes the pointers (_ptr: a contiguous
# CUDA tensor on the call's device).

def _fits(t, nbytes: int, name: str, dtype=None) -> None:
    if dtype is not None and t.dtype != dtype:
        raise ValueError(f"{name} must be {dtype}")
    have = t.numel() * t.element_size()
    if have < nbytes:
        raise ValueError(f"{name} holds {have} bytes; the call needs {nbytes}")


def _check_stored(packed, norms, rows: int, cols: int, bits: int, group_size: int) -> None:
    torch = _torch()
    _fits(packed, packed_bytes(rows, cols, bits, group_size), "packed", torch.uint8)
    _fits(norms, norm_bytes(rows, cols, group_size), "norms", torch.float16)


def _check_x(x, cols: int) -> None:
    torch = _torch()
    if x.dim() != 2 or x.shape[1] != cols:
        raise ValueError(f"x must be [batch, {cols}]")
    _fits(x, 0, "x", torch.bfloat16)


def _ptr(t, name: str, device) -> int:
    ptr = _dev_ptr(t, name)
    if t.device != device:
        raise ValueError(f"{name} must be on {device}")
    return ptr


def _cb_ptr(cb, device) -> int | None:
    if cb is None:
        return None
    torch = _torch()
    if cb.dtype != torch.float32 or not cb.is_cuda or cb.device != device:
        raise ValueError("codebook must be a float32 CUDA tensor on the same device")
    return _dev_ptr(cb, "codebook")


def empty_packed(rows: int, cols: int, bits: int, device, group_size: int = GROUP_SIZE):
    torch = _torch()
    G = -(-cols // group_size)
    return (torch.empty((rows, G, group_size * field_bits(bits) // 8), dtype=torch.uint8,
                        device=device),
            torch.empty((rows, G), dtype=torch.float16, device=device))


def quantize(w, bits: int, group_size: int = GROUP_SIZE, codebook=None, out=None):
    """cq_quantize on a 2-D bf16/fp32 CUDA tensor -> (packed uint8, norms float16)."""
    torch = _torch()
    if w.dim() != 2:
        raise ValueError("w must be 2-D [rows, cols]")
    if w.dtype == torch.bfloat16:
        dt = CQ_BF16
    elif w.dtype == torch.float32:
        dt = CQ_F32
    else:
        raise ValueError("w must be bfloat16 or float32")
    rows, cols = w.shape
    packed, norms = out if out is not None else empty_packed(rows, cols, bits, w.device, group_size)
    _check_stored(packed, norms, rows, cols, bits, group_size)
    with torch.cuda.device(w.device):
        _check(lib().cq_quantize(_dev_ptr(w, "w"), dt, rows, cols, bits, group_size,
                                 _cb_ptr(codebook, w.device), _ptr(packed, "packed", w.device),
                                 _ptr(norms, "norms", w.device), _stream(w.device)), "cq_quantize")
    return packed, norms


class _QuantizeJob(ctypes.Structure):  # cq_quantize_job
    _fields_ = [("w", ctypes.c_void_p), ("rows", ctypes.c_longlong), ("cols", ctypes.c_longlong),
                ("packed_out", ctypes.c_void_p), ("norms_out", ctypes.c_void_p)]


class _DequantizeJob(ctypes.Structure):  # cq_dequantize_job
    _fields_ = [("packed", ctypes.c_void_p), ("norms", ctypes.c_void_p), ("rows", ctypes.c_longlong),
                ("cols", ctypes.c_longlong), ("out", ctypes.c_void_p)]


def quantize_batch(ws, bits: int, group_size: int = GROUP_SIZE, codebook=None, outs=None):
    """cq_quantize_batch on a list of 2-D CUDA tensors of one dtype (bf16 or fp32) on one
    device -> list of (packed, norms).  `outs`, if given, is a list of (packed, norms)."""
    torch = _torch()
    if not ws:
        return []
    dev, dtype = ws[0].device, ws[0].dtype
    if dtype == torch.bfloat16:
        dt = CQ_BF16
    elif dtype == torch.float32:
        dt = CQ_F32
    else:
        raise ValueError("tensors must be bfloat16 or float32")
    if outs is not None and len(outs) != len(ws):
        raise ValueError("one (packed, norms) pair per tensor")
    jobs = (_QuantizeJob * len(ws))()
    res = []
    for k, w in enumerate(ws):
        if w.dim() != 2 or w.dtype != dtype or w.device != dev:
            raise ValueError("tensors must be 2-D, of one dtype, on one device")
        rows, cols = w.shape
        packed, norms = outs[k] if outs is not None else empty_packed(rows, cols, bits, dev, group_size)
        _check_stored(packed, norms, rows, cols, bits, group_size)
        jobs[k] = _QuantizeJob(_dev_ptr(w, "w"), rows, cols, _ptr(packed, "packed", dev), _ptr(norms, "norms", dev))
        res.append((packed, norms))
    with torch.cuda.device(dev):
        _check(lib().cq_quantize_batch(ctypes.cast(jobs, ctypes.c_void_p), len(ws), dt, bits, group_size,
                                       _cb_ptr(codebook, dev), _stream(dev)), "cq_quantize_batch")
    return res


def dequantize_batch(items, bits: int, group_size: int = GROUP_SIZE, codebook=None,
                     out_dtype=None, outs=None):
    """cq_dequantize_batch on a list of (packed, norms, rows, cols) on one device -> list of
    W_hat tensors (bfloat16 by default, or float32; `outs` gives them)."""
    torch = _torch()
    if not items:
        return []
    dev = items[0][0].device
    if outs is None:
        out_dtype = torch.bfloat16 if out_dtype is None else out_dtype
        outs = [torch.empty((r, c), dtype=out_dtype, device=dev) for _, _, r, c in items]
    if len(outs) != len(items):
        raise ValueError("one output per item")
    dtype = outs[0].dtype
    if dtype == torch.bfloat16:
        dt = CQ_BF16
    elif dtype == torch.float32:
        dt = CQ_F32
    else:
        raise ValueError("out dtype must be bfloat16 or float32")
    jobs = (_DequantizeJob * len(items))()
    for k, ((packed, norms, rows, cols), out) in enumerate(zip(items, outs)):
        _check_stored(packed, norms, rows, cols, bits, group_size)
        _fits(out, rows * cols * out.element_size(), "out", dtype)
        jobs[k] = _DequantizeJob(_ptr(packed, "packed", dev), _ptr(norms, "norms", dev), rows, cols,
                                 _ptr(out, "out", dev))
    with torch.cuda.device(dev):
        _check(lib().cq_dequantize_batch(ctypes.cast(jobs, ctypes.c_void_p), len(items), bits,
                                         group_size, _cb_ptr(codebook, dev), dt, _stream(dev)),
               "cq_dequantize_batch")
    return outs


class _GemvJob(ctypes.Structure):  # cq_gemv_job
    _fields_ = [("packed", ctypes.c_void_p), ("norms", ctypes.c_void_p), ("rows", ctypes.c_longlong),
                ("cols", ctypes.c_longlong), ("x", ctypes.c_void_p), ("batch", ctypes.c_int),
                ("y", ctypes.c_void_p), ("workspace", ctypes.c_void_p), ("workspace_bytes", ctypes.c_size_t)]


def dequant_gemv_batch(items, bits: int, group_size: int = GROUP_SIZE, codebook=None,
                       workspaces=None, ys=None):
    """cq_dequant_gemv_batch on a list of (packed, norms, rows, cols, x) on one device ->
    list of y [batch, rows] fp32.  `workspaces` / `ys`, if given, are lists of tensors (each
    job needs its own workspace)."""
    torch = _torch()
    if not items:
        return []
    dev = items[0][0].device
    if (ys is not None and len(ys) != len(items)) or (workspaces is not None and len(workspaces) != len(items)):
        raise ValueError("one y and one workspace per product")
    jobs = (_GemvJob * len(items))()
    out = []
    keep = []  # every job's workspace stays allocated until the launches are enqueued
    for k, (packed, norms, rows, cols, x) in enumerate(items):
        if x.dim() == 1:
            x = x.unsqueeze(0)
        batch = x.shape[0]
        _check_x(x, cols)
        _check_stored(packed, norms, rows, cols, bits, group_size)
        y = ys[k] if ys is not None else torch.empty((batch, rows), dtype=torch.float32, device=dev)
        _fits(y, 4 * batch * rows, "y", torch.float32)
        wsb = gemv_workspace_bytes(cols, batch)
        ws = workspaces[k] if workspaces is not None else torch.empty(max(wsb, 16), dtype=torch.uint8, device=dev)
        keep.append(ws)
        jobs[k] = _GemvJob(_ptr(packed, "packed", dev), _ptr(norms, "norms", dev), rows, cols,
                           _ptr(x, "x", dev), batch, _ptr(y, "y", dev), _ptr(ws, "workspace", dev),
                           ws.numel() * ws.element_size())
        out.append(y)
    with torch.cuda.device(dev):
        _check(lib().cq_dequant_gemv_batch(ctypes.cast(jobs, ctypes.c_void_p), len(items), bits,
                                           group_size, _cb_ptr(codebook, dev), _stream(dev)),
               "cq_dequant_gemv_batch")
    return out


def _dtype_code(dtype, what: str) -> int:
    torch = _torch()
    if dtype == torch.bfloat16:
        return CQ_BF16
    if dtype == torch.float32:
        return CQ_F32
    raise ValueError(f"{what} must be bfloat16 or float32")


def fake_quantize(w, bits: int, group_size: int = GROUP_SIZE, codebook=None, out_dtype=None,
                  out=None, stored=None):
    """cq_fake_quantize -> W_hat = dequantize(quantize(w)), the tensor the pages' cq_quantize
    returns (same dtype as w unless `out_dtype` / `out` say otherwise; `out=w` works in place).
    `stored`, if given, is the (packed, norms) pair that receives the stored form."""
    torch = _torch()
    if w.dim() != 2:
        raise ValueError("w must be 2-D [rows, cols]")
    wt = _dtype_code(w.dtype, "w")
    rows, cols = w.shape
    if out is None:
        out = torch.empty((rows, cols), dtype=w.dtype if out_dtype is None else out_dtype, device=w.device)
    ot = _dtype_code(out.dtype, "out")
    if tuple(out.shape) != (rows, cols):
        raise ValueError("out must have the shape of w")
    packed, norms = stored if stored is not None else empty_packed(rows, cols, bits, w.device, group_size)
    _check_stored(packed, norms, rows, cols, bits, group_size)
    dev = w.device
    with torch.cuda.device(dev):
        _check(lib().cq_fake_quantize(_dev_ptr(w, "w"), wt, rows, cols, bits, group_size,
                                      _cb_ptr(codebook, dev), _ptr(packed, "packed", dev),
                                      _ptr(norms, "norms", dev), _ptr(out, "out", dev), ot,
                                      _stream(dev)), "cq_fake_quantize")
    return out


class _FakeQuantizeJob(ctypes.Structure):  # cq_fake_quantize_job
    _fields_ = [("w", ctypes.c_void_p), ("rows", ctypes.c_longlong), ("cols", ctypes.c_longlong),
                ("packed_out", ctypes.c_void_p), ("norms_out", ctypes.c_void_p), ("out", ctypes.c_void_p)]


def fake_quantize_batch(ws, bits: int, group_size: int = GROUP_SIZE, codebook=None, out_dtype=None,
                        outs=None, stored=None):
    """cq_fake_quantize_batch on a list of 2-D CUDA tensors of one dtype on one device ->
    list of W_hat tensors (`outs` may be `ws` itself for in-place fake quantisation).
    `stored`, if given, is a list of (packed, norms) pairs receiving the stored forms."""
    torch = _torch()
    if not ws:
        return []
    dev = ws[0].device
    wt = _dtype_code(ws[0].dtype, "w")
    if outs is None:
        odt = ws[0].dtype if out_dtype is None else out_dtype
        outs = [torch.empty(tuple(w.shape), dtype=odt, device=dev) for w in ws]
    if len(outs) != len(ws) or (stored is not None and len(stored) != len(ws)):
        raise ValueError("one output (and one stored pair) per tensor")
    ot = _dtype_code(outs[0].dtype, "out")
    jobs = (_FakeQuantizeJob * len(ws))()
    keep = []  # intermediate buffers stay allocated until the launches are enqueued
    for k, (w, out) in enumerate(zip(ws, outs)):
        if w.dim() != 2 or w.dtype != ws[0].dtype or w.device != dev:
            raise ValueError("tensors must be 2-D, of one dtype, on one device")
        if out.dtype != outs[0].dtype or out.device != dev or tuple(out.shape) != tuple(w.shape):
            raise ValueError("outputs must match their inputs' shapes and share one dtype")
        rows, cols = w.shape
        packed, norms = stored[k] if stored is not None else empty_packed(rows, cols, bits, dev, group_size)
        keep.append((packed, norms))
        _check_stored(packed, norms, rows, cols, bits, group_size)
        jobs[k] = _FakeQuantizeJob(_dev_ptr(w, "w"), rows, cols, _ptr(packed, "packed", dev),
                                   _ptr(norms, "norms", dev), _ptr(out, "out", dev))
    with torch.cuda.device(dev):
        _check(lib().cq_fake_quantize_batch(ctypes.cast(jobs, ctypes.c_void_p), len(ws), wt, bits,
                                            group_size, _cb_ptr(codebook, dev), ot, _stream(dev)),
               "cq_fake_quantize_batch")
    return outs


def dequantize(packed, norms, rows: int, cols: int, bits: int, group_size: int = GROUP_SIZE,
               codebook=None, out_dtype=None, out=None):
    """cq_dequantize -> W_hat [rows, cols] (bfloat16 by default, or float32)."""
    torch = _torch()
    if out is None:
        out_dtype = torch.bfloat16 if out_dtype is None else out_dtype
        out = torch.empty((rows, cols), dtype=out_dtype, device=packed.device)
    if out.dtype == torch.bfloat16:
        dt = CQ_BF16
    elif out.dtype == torch.float32:
        dt = CQ_F32
    else:
        raise ValueError("out dtype must be bfloat16 or float32")
    dev = packed.device
    _check_stored(packed, norms, rows, cols, bits, group_size)
    _fits(out, rows * cols * out.element_size(), "out")
    with torch.cuda.device(dev):
        _check(lib().cq_dequantize(_ptr(packed, "packed", dev), _ptr(norms, "norms", dev), rows, cols,
                                   bits, group_size, _cb_ptr(codebook, dev), _ptr(out, "out", dev), dt,
                                   _stream(dev)), "cq_dequantize")
    return out


def dequant_gemv(packed, norms, rows: int, cols: int, bits: int, x, group_size: int = GROUP_SIZE,
                 codebook=None, workspace=None, y=None):
    """cq_dequant_gemv: y [batch, rows] fp32 = W_hat x for x bf16 [batch, cols]."""
    torch = _torch()
    if x.dim() == 1:
        x = x.unsqueeze(0)
    if x.dtype != torch.bfloat16:
        raise ValueError("x must be bfloat16")
    batch = x.shape[0]
    dev = packed.device
    _check_x(x, cols)
    _check_stored(packed, norms, rows, cols, bits, group_size)
    if y is None:
        y = torch.empty((batch, rows), dtype=torch.float32, device=dev)
    _fits(y, 4 * batch * rows, "y", torch.float32)
    ws_bytes = gemv_workspace_bytes(cols, batch)
    if workspace is None:
        workspace = torch.empty(max(ws_bytes, 16), dtype=torch.uint8, device=dev)
    with torch.cuda.device(dev):
        _check(lib().cq_dequant_gemv(_ptr(packed, "packed", dev), _ptr(norms, "norms", dev), rows, cols,
                                     bits, group_size, _cb_ptr(codebook, dev), _ptr(x, "x", dev), batch,
                                     _ptr(y, "y", dev), _ptr(workspace, "workspace", dev),
                                     workspace.numel() * workspace.element_size(),
                                     _stream(dev)), "cq_dequant_gemv")
    return y


def dequant_gemv_static(packed, norms, rows: int, cols: int, bits: int, x,
                        group_size: int = GROUP_SIZE, codebook=None, y=None):
    """cq_dequant_gemv_static: the GEMV with the library's built-in scratch (cols <= 32768),
    for callers that must not allocate device memory."""
    torch = _torch()
    if x.dim() == 1:
        x = x.unsqueeze(0)
    batch = x.shape[0]
    dev = packed.device
    _check_x(x, cols)
    _check_stored(packed, norms, rows, cols, bits, group_size)
    if y is None:
        y = torch.empty((batch, rows), dtype=torch.float32, device=dev)
    _fits(y, 4 * batch * rows, "y", torch.float32)
    with torch.cuda.device(dev):
        _check(lib().cq_dequant_gemv_static(_ptr(packed, "packed", dev), _ptr(norms, "norms", dev),
                                            rows, cols, bits, group_size, _cb_ptr(codebook, dev),
                                            _ptr(x, "x", dev), batch, _ptr(y, "y", dev),
                                            _stream(dev)), "cq_dequant_gemv_static")
    return y
