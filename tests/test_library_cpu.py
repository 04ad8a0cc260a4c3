"""CPU-only checks of libcq: it builds, loads, exports what include/cq.h declares, its host
routines agree with the oracle, and bad arguments are rejected before anything runs."""
import ctypes
import os
import re

import numpy as np
import pytest

import hadamard_codebook_bit_b200 as cq
from hadamard_codebook_bit_b200 import build as cq_build

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


@pytest.fixture(scope="module")
def L():
    cq_build.build()
    return cq.lib()


def declared_functions():
    text = open(os.path.join(ROOT, "include", "cq.h")).read()
    text = re.sub(r"/\*.*?\*/", "", text, flags=re.S)
    return sorted(set(re.findall(r"\b(cq_[a-z0-9_]+)\s*\(", text)))


def test_header_declares_the_binding_exports():
    assert declared_functions() == sorted(cq.EXPORTS)


def test_library_exports_every_declared_symbol(L):
    for name in declared_functions():
        assert hasattr(L, name), name
    # and the ELF dynamic table lists them as defined functions
    import subprocess
    out = subprocess.run(["nm", "-D", "--defined-only", cq.LIB_PATH], capture_output=True,
                         text=True, check=True).stdout
    for name in declared_functions():
        assert re.search(rf"\bT {name}$", out, flags=re.M), name


def test_status_strings(L):
    for s in range(6):
        assert L.cq_status_string(s).decode().startswith("CQ")
    assert b"unknown" in L.cq_status_string(99)
    assert L.cq_version() == 10000


@pytest.mark.parametrize("bits", [0, 2, 3, 4])
@pytest.mark.parametrize("seed", [0, 7])
def test_library_codebook_equals_oracle(oracle_lib, bits, seed, L):
    if bits == 0 and seed:
        pytest.skip("ternary ignores the seed")
    ours = cq.codebook(bits, 128, seed)
    ref = oracle_lib.codebook(bits, 128, seed)
    assert ours.dtype == np.float32
    assert np.array_equal(ours, ref)


def test_codebook_other_group_sizes(oracle_lib, L):
    for g in (8, 64, 256, 4096):
        assert np.array_equal(cq.codebook(2, g), oracle_lib.codebook(2, g))


def test_codebook_rejects_bad_arguments(L):
    out = np.zeros(16, np.float32)
    p = out.ctypes.data_as(ctypes.c_void_p)
    for bits, g, seed in [(1, 128, 0), (5, 128, 0), (2, 96, 0), (2, 4, 0), (2, 8192, 0),
                          (2, 128, 2**32)]:
        assert L.cq_codebook(bits, g, seed, p, None) == 1
    assert L.cq_codebook(2, 128, 0, None, None) == 1


@pytest.mark.parametrize("rows,cols,bits", [(256, 512, 2), (768, 1000, 3), (1, 1, 0),
                                            (4096, 11008, 4), (3, 129, 2)])
def test_byte_counts_match_oracle(oracle_lib, rows, cols, bits, L):
    assert cq.packed_bytes(rows, cols, bits) == oracle_lib.packed_bytes(rows, cols, bits)
    assert cq.norm_bytes(rows, cols) == oracle_lib.norm_bytes(rows, cols)


def test_byte_counts_edge_cases(L):
    assert cq.packed_bytes(0, 5, 2) == 0 and cq.norm_bytes(5, 0) == 0
    assert cq.packed_bytes(-1, 5, 2) == 0 and cq.packed_bytes(5, 5, 7) == 0
    def ws(G):  # B-operand fragments, per-column exponents, one 48-byte codeword table
        return -(-(G * 2080 + 48) // 256) * 256
    assert cq.gemv_workspace_bytes(4096, 1) == ws(32) == cq.gemv_workspace_bytes(4096, 8)
    assert cq.gemv_workspace_bytes(11008, 8) == ws(86)
    assert cq.gemv_workspace_bytes(1, 3) == ws(1)
    assert cq.gemv_workspace_bytes(4096, 9) == 2 * ws(32) == cq.gemv_workspace_bytes(4096, 16)
    assert cq.gemv_workspace_bytes(4096, 64) == 8 * ws(32)
    assert cq.gemv_workspace_bytes(4096, 65) == 0 and cq.gemv_workspace_bytes(4096, 0) == 0


# ------------------------------------------------------------------------------------------
# argument validation: every call below must fail on the host, before any CUDA call
# ------------------------------------------------------------------------------------------

A = 4096  # a fake, 16-byte aligned "device address": never dereferenced, nothing launches


def test_quantize_rejects(L):
    q = L.cq_quantize
    assert q(A, 2, 4, 128, 2, 128, None, A, A, None) == 1      # bad dtype
    assert q(A, 1, -1, 128, 2, 128, None, A, A, None) == 1     # negative rows
    assert q(A, 1, 4, 128, 1, 128, None, A, A, None) == 1      # bits 1
    assert q(A, 1, 4, 128, 5, 128, None, A, A, None) == 1      # bits 5
    assert q(A, 1, 4, 128, 2, 100, None, A, A, None) == 1      # group not a power of two
    assert q(A, 1, 4, 128, 2, 64, None, A, A, None) == 2       # valid but unsupported
    assert q(None, 1, 4, 128, 2, 128, None, A, A, None) == 1   # null input
    assert q(A, 1, 4, 128, 2, 128, None, None, A, None) == 1   # null packed
    assert q(A + 8, 1, 4, 128, 2, 128, None, A, A, None) == 4  # misaligned
    assert q(A, 1, 4, 128, 2, 128, None, A, A + 2, None) == 4
    assert q(A, 1, 1 << 40, 1 << 20, 2, 128, None, A, A, None) == 1  # absurd size


def test_empty_shapes_are_no_ops(L):
    assert L.cq_quantize(None, 1, 0, 128, 2, 128, None, None, None, None) == 0
    assert L.cq_quantize(None, 0, 7, 0, 4, 128, None, None, None, None) == 0
    assert L.cq_dequantize(None, None, 0, 64, 3, 128, None, None, 1, None) == 0
    assert L.cq_dequant_gemv(None, None, 0, 64, 2, 128, None, None, 1, None, None, 0, None) == 0


def test_dequantize_rejects(L):
    d = L.cq_dequantize
    assert d(A, A, 4, 128, 2, 128, None, A, 3, None) == 1       # bad out dtype
    assert d(A, A, 4, 128, 6, 128, None, A, 1, None) == 1
    assert d(A, A, 4, 128, 2, 256, None, A, 1, None) == 2
    assert d(A, None, 4, 128, 2, 128, None, A, 1, None) == 1
    assert d(A, A, 4, 128, 2, 128, None, A + 4, 1, None) == 4


def test_gemv_rejects(L):
    g = L.cq_dequant_gemv
    ws = cq.gemv_workspace_bytes(256, 1)
    assert g(A, A, 4, 256, 2, 128, None, A, 0, A, A, ws, None) == 1    # batch 0
    assert g(A, A, 4, 256, 2, 128, None, A, 65, A, A, ws, None) == 1   # batch 65
    ws64 = cq.gemv_workspace_bytes(256, 64)
    assert ws64 == 8 * cq.gemv_workspace_bytes(256, 8) and cq.gemv_workspace_bytes(256, 9) == 2 * ws
    assert g(A, A, 4, 256, 2, 128, None, A, 9, A, A, ws, None) == 5    # batch 9 needs two blocks
    assert g(A, A, 4, 256, 2, 128, None, A, 64, A, A, ws64 - 1, None) == 5
    assert g(A, A, 4, 256, 2, 128, None, None, 1, A, A, ws, None) == 1  # null x
    assert g(A, A, 4, 256, 2, 128, None, A, 1, A, None, ws, None) == 5  # no workspace
    assert g(A, A, 4, 256, 2, 128, None, A, 1, A, A, ws - 1, None) == 5
    assert g(A, A, 4, 256, 2, 128, None, A, 1, A + 4, A, ws, None) == 4
    assert g(A, A, 4, 256, 2, 32, None, A, 1, A, A, ws, None) == 2


def _qjobs(*jobs):
    arr = (cq._QuantizeJob * max(1, len(jobs)))()
    for k, j in enumerate(jobs):
        arr[k] = cq._QuantizeJob(*j)
    return ctypes.cast(arr, ctypes.c_void_p), arr


def _dqjobs(*jobs):
    arr = (cq._DequantizeJob * max(1, len(jobs)))()
    for k, j in enumerate(jobs):
        arr[k] = cq._DequantizeJob(*j)
    return ctypes.cast(arr, ctypes.c_void_p), arr


def test_quantize_batch_rejects_before_launching(L):
    q = L.cq_quantize_batch
    good = (A, 4, 128, A, A)
    p, _k = _qjobs(good, good)
    assert q(p, -1, 1, 2, 128, None, None) == 1                 # negative count
    assert q(None, 1, 1, 2, 128, None, None) == 1               # no job array
    assert q(p, 2, 2, 2, 128, None, None) == 1                  # bad dtype
    assert q(p, 2, 1, 1, 128, None, None) == 1                  # bits 1
    assert q(p, 2, 1, 2, 64, None, None) == 2                   # valid but unsupported group
    p, _k = _qjobs(good, (A, -1, 128, A, A))
    assert q(p, 2, 1, 2, 128, None, None) == 1                  # second job: negative rows
    p, _k = _qjobs(good, (A, 4, 128, None, A))
    assert q(p, 2, 1, 2, 128, None, None) == 1                  # second job: null packed
    p, _k = _qjobs((A + 8, 4, 128, A, A), good)
    assert q(p, 2, 1, 2, 128, None, None) == 4                  # first job misaligned
    assert q(None, 0, 1, 2, 128, None, None) == 0               # nothing to do
    p, _k = _qjobs((None, 0, 128, None, None), (None, 7, 0, None, None))
    assert q(p, 2, 1, 2, 128, None, None) == 0                  # only empty jobs


def test_dequantize_batch_rejects_before_launching(L):
    d = L.cq_dequantize_batch
    good = (A, A, 4, 128, A)
    p, _k = _dqjobs(good, good)
    assert d(p, -1, 2, 128, None, 1, None) == 1
    assert d(None, 2, 2, 128, None, 1, None) == 1
    assert d(p, 2, 2, 128, None, 3, None) == 1                  # bad out dtype
    assert d(p, 2, 6, 128, None, 1, None) == 1                  # bits 6
    p, _k = _dqjobs(good, (A, None, 4, 128, A))
    assert d(p, 2, 2, 128, None, 1, None) == 1                  # null norms
    p, _k = _dqjobs(good, (A, A, 4, 128, A + 4))
    assert d(p, 2, 2, 128, None, 1, None) == 4                  # misaligned out
    p, _k = _dqjobs((None, None, 0, 64, None))
    assert d(p, 1, 3, 128, None, 1, None) == 0                  # only an empty job


def test_gemv_batch_rejects_before_launching(L):
    g = L.cq_dequant_gemv_batch
    ws = cq.gemv_workspace_bytes(256, 1)

    def jobs(*js):
        arr = (cq._GemvJob * len(js))()
        for k, j in enumerate(js):
            arr[k] = cq._GemvJob(*j)
        return ctypes.cast(arr, ctypes.c_void_p), arr

    good = (A, A, 4, 256, A, 1, A, A, ws)
    p, _k = jobs(good, good)
    assert g(p, -1, 2, 128, None, None) == 1
    assert g(None, 2, 2, 128, None, None) == 1
    assert g(p, 2, 5, 128, None, None) == 1                          # bits 5
    p, _k = jobs(good, (A, A, 4, 256, A, 65, A, A, 8 * ws))
    assert g(p, 2, 2, 128, None, None) == 1                          # batch 65
    p, _k = jobs(good, (A, A, 4, 256, A, 9, A, A, ws))
    assert g(p, 2, 2, 128, None, None) == 5                          # batch 9: two blocks of workspace
    p, _k = jobs(good, (A, A, 4, 256, A, 1, A, A, ws - 1))
    assert g(p, 2, 2, 128, None, None) == 5                          # workspace too small
    p, _k = jobs(good, (A, A, 4, 256, A, 1, A + 4, A, ws))
    assert g(p, 2, 2, 128, None, None) == 4                          # misaligned y
    p, _k = jobs((None, None, 0, 256, None, 1, None, None, 0))
    assert g(p, 1, 2, 128, None, None) == 0                          # rows == 0: nothing to do


def _fjobs(*jobs):
    arr = (cq._FakeQuantizeJob * max(1, len(jobs)))()
    for k, j in enumerate(jobs):
        arr[k] = cq._FakeQuantizeJob(*j)
    return ctypes.cast(arr, ctypes.c_void_p), arr


def test_fake_quantize_rejects_before_launching(L):
    f = L.cq_fake_quantize
    assert f(A, 2, 4, 128, 2, 128, None, A, A, A, 1, None) == 1       # bad w dtype
    assert f(A, 1, 4, 128, 2, 128, None, A, A, A, 2, None) == 1       # bad out dtype
    assert f(A, 1, 4, 128, 5, 128, None, A, A, A, 1, None) == 1       # bits 5
    assert f(A, 1, 4, 128, 2, 64, None, A, A, A, 1, None) == 2        # unsupported group
    assert f(A, 1, 4, 128, 2, 128, None, A, A, None, 1, None) == 1    # null out
    assert f(A, 1, 4, 128, 2, 128, None, None, A, A, 1, None) == 1    # null packed
    assert f(A, 1, 4, 128, 2, 128, None, A, A, A + 2, 1, None) == 4   # misaligned out
    assert f(A, 1, 4, 128, 2, 128, None, A, A + 2, A, 1, None) == 4   # misaligned norms
    assert f(A, 1, 4, 128, 2, 128, A + 2, A, A, A, 1, None) == 4      # misaligned codebook
    assert f(None, 1, 0, 128, 2, 128, None, None, None, None, 1, None) == 0  # empty
    b = L.cq_fake_quantize_batch
    good = (A, 4, 128, A, A, A)
    p, _k = _fjobs(good, good)
    assert b(p, -1, 1, 2, 128, None, 1, None) == 1
    assert b(None, 1, 1, 2, 128, None, 1, None) == 1
    assert b(p, 2, 1, 2, 128, None, 3, None) == 1                     # bad out dtype
    assert b(p, 2, 0, 1, 128, None, 1, None) == 1                     # bits 1
    p, _k = _fjobs(good, (A, 4, 128, A, A, None))
    assert b(p, 2, 1, 2, 128, None, 1, None) == 1                     # second job: null out
    p, _k = _fjobs(good, (A, 4, 128, A, A, A + 8))
    assert b(p, 2, 1, 2, 128, None, 1, None) == 4                     # second job: misaligned out
    p, _k = _fjobs((None, 0, 128, None, None, None), (None, 3, 0, None, None, None))
    assert b(p, 2, 1, 4, 128, None, 0, None) == 0                     # only empty jobs
    assert b(None, 0, 1, 2, 128, None, 1, None) == 0                  # nothing to do


def test_binding_refuses_cpu_tensors(L):
    torch = pytest.importorskip("torch")
    with pytest.raises(ValueError):
        cq.quantize(torch.zeros(4, 128, dtype=torch.bfloat16), 2)
    with pytest.raises(ValueError):
        cq.fake_quantize(torch.zeros(4, 128, dtype=torch.bfloat16), 2)
    with pytest.raises(ValueError):
        cq.fake_quantize(torch.zeros(4, 128, dtype=torch.float16), 2)  # unsupported dtype
    with pytest.raises(ValueError):
        cq.fake_quantize_batch([torch.zeros(4, 128, dtype=torch.bfloat16)], 2)
    with pytest.raises(ValueError):
        cq.fake_quantize_batch([torch.zeros(4, 128, dtype=torch.bfloat16)], 2,
                               outs=[torch.zeros(4, 64, dtype=torch.bfloat16)])  # shape mismatch


def test_binding_checks_buffer_sizes_before_any_call(L):
    """The C ABI takes plain pointers, so the binding checks every buffer against the sizes
    the call will touch (CPU tensors: the size checks come first, then 'must be a CUDA
    tensor' for correctly sized ones)."""
    torch = pytest.importorskip("torch")
    rows, cols, bits = 4, 300, 2
    G = 3
    w = torch.zeros(rows, cols, dtype=torch.bfloat16)
    ok_p = torch.zeros(rows, G, 32, dtype=torch.uint8)
    ok_n = torch.zeros(rows, G, dtype=torch.float16)
    small_p = torch.zeros(rows, G, 31, dtype=torch.uint8)
    with pytest.raises(ValueError, match="packed holds"):
        cq.quantize(w, bits, out=(small_p, ok_n))
    with pytest.raises(ValueError, match="norms must be"):
        cq.quantize(w, bits, out=(ok_p, ok_n.view(torch.int16)))
    with pytest.raises(ValueError, match="CUDA tensor|cuda device"):
        cq.quantize(w, bits, out=(ok_p, ok_n))
    with pytest.raises(ValueError, match="packed holds"):
        cq.dequantize(small_p, ok_n, rows, cols, bits)
    with pytest.raises(ValueError, match="out holds"):
        cq.dequantize(ok_p, ok_n, rows, cols, bits, out=torch.zeros(rows, cols - 1, dtype=torch.bfloat16))
    with pytest.raises(ValueError, match="CUDA tensor|cuda device"):
        cq.dequantize(ok_p, ok_n, rows, cols, bits, out=torch.zeros(rows, cols, dtype=torch.bfloat16))
    x = torch.zeros(2, cols, dtype=torch.bfloat16)
    with pytest.raises(ValueError, match=r"x must be \[batch, 300\]"):
        cq.dequant_gemv(ok_p, ok_n, rows, cols, bits, torch.zeros(2, cols + 1, dtype=torch.bfloat16))
    with pytest.raises(ValueError, match="y holds"):
        cq.dequant_gemv(ok_p, ok_n, rows, cols, bits, x, y=torch.zeros(2, rows - 1))
    with pytest.raises(ValueError, match="CUDA tensor|cuda device"):
        cq.dequant_gemv(ok_p, ok_n, rows, cols, bits, x, y=torch.zeros(2, rows))
    with pytest.raises(ValueError, match="y holds"):
        cq.dequant_gemv_static(ok_p, ok_n, rows, cols, bits, x, y=torch.zeros(1, rows))
    with pytest.raises(ValueError, match="norms holds"):
        cq.dequant_gemv_batch([(ok_p, ok_n[:, :2].contiguous(), rows, cols, x)], bits)
    with pytest.raises(ValueError, match="one y and one workspace"):
        cq.dequant_gemv_batch([(ok_p, ok_n, rows, cols, x)], bits, ys=[])
    with pytest.raises(ValueError, match="one output per item"):
        cq.dequantize_batch([(ok_p, ok_n, rows, cols)], bits, outs=[])
    with pytest.raises(ValueError, match="one .packed, norms. pair per tensor"):
        cq.quantize_batch([w, w], bits, outs=[(ok_p, ok_n)])
    with pytest.raises(ValueError, match="packed holds"):
        cq.fake_quantize(w, bits, stored=(small_p, ok_n))
    with pytest.raises(ValueError, match="one output"):
        cq.fake_quantize_batch([w, w], bits, outs=[w])


class _FakeLib:
    """Stands in for libcq in the marshalling test: records each call, launches nothing."""

    def __init__(self, real):
        self.real = real
        self.calls = []

    def __getattr__(self, name):
        if name in ("cq_packed_bytes", "cq_norm_bytes", "cq_gemv_workspace_bytes", "cq_status_string"):
            return getattr(self.real, name)

        def call(*args):
            self.calls.append((name, args))
            return 0
        return call


def test_binding_marshals_valid_calls(L, monkeypatch):
    """Every binding entry point accepts the shapes the GPU tests and the bench use (CPU
    tensors stand in for device ones; the fake library records the calls)."""
    torch = pytest.importorskip("torch")
    import contextlib
    fake = _FakeLib(L)
    monkeypatch.setattr(cq, "lib", lambda: fake)
    monkeypatch.setattr(cq, "_dev_ptr", lambda t, name: t.data_ptr())
    monkeypatch.setattr(cq, "_stream", lambda device: 0)
    monkeypatch.setattr(torch.cuda, "device", lambda d: contextlib.nullcontext())
    bf = torch.bfloat16
    for rows, cols, bits in ((37, 1000, 2), (4, 128, 0), (3, 129, 3), (5, 8, 4), (0, 128, 2), (7, 0, 2)):
        w = torch.zeros(rows, cols, dtype=bf)
        packed, norms = cq.quantize(w, bits)
        cq.quantize(w.float(), bits, out=(packed, norms))
        cq.dequantize(packed, norms, rows, cols, bits)
        cq.dequantize(packed, norms, rows, cols, bits, out=torch.zeros(rows, cols))
        cq.fake_quantize(w, bits)
        cq.fake_quantize(w, bits, out=w, stored=(packed, norms))
        cq.fake_quantize(w, bits, out_dtype=torch.float32)
        for batch in (1, 8, 9, 64):
            x = torch.zeros(batch, cols, dtype=bf)
            cq.dequant_gemv(packed, norms, rows, cols, bits, x)
            cq.dequant_gemv(packed, norms, rows, cols, bits, x, y=torch.zeros(batch, rows),
                            workspace=torch.zeros(cq.gemv_workspace_bytes(cols, batch) or 16, dtype=torch.uint8))
            cq.dequant_gemv_static(packed, norms, rows, cols, bits, x)
        cq.dequant_gemv(packed, norms, rows, cols, bits, torch.zeros(cols, dtype=bf))  # 1-D x
    # batched calls, including views of one flat buffer as the bench lays the set out
    shapes = [(64, 256), (11, 1000), (0, 128), (3, 11008)]
    ws = [torch.zeros(r, c, dtype=bf) for r, c in shapes]
    q = cq.quantize_batch(ws, 2)
    flat_p = torch.zeros(sum(p.numel() for p, _ in q), dtype=torch.uint8)
    flat_n = torch.zeros(sum(n.numel() for _, n in q), dtype=torch.float16)
    views, op, on = [], 0, 0
    for p, n in q:
        views.append((flat_p[op:op + p.numel()].view(p.shape), flat_n[on:on + n.numel()].view(n.shape)))
        op += p.numel()
        on += n.numel()
    cq.quantize_batch(ws, 2, outs=views)
    items = [(p, n, r, c) for (p, n), (r, c) in zip(views, shapes)]
    cq.dequantize_batch(items, 2)
    cq.dequantize_batch(items, 2, outs=[torch.zeros(r, c) for r, c in shapes])
    cq.dequant_gemv_batch([(p, n, r, c, torch.zeros(1 + k, c, dtype=bf)) for k, (p, n, r, c) in enumerate(items)], 2)
    cq.fake_quantize_batch(ws, 2)
    cq.fake_quantize_batch(ws, 2, outs=ws, stored=views)
    names = {n for n, _ in fake.calls}
    assert names == {"cq_quantize", "cq_dequantize", "cq_fake_quantize", "cq_dequant_gemv",
                     "cq_dequant_gemv_static", "cq_quantize_batch", "cq_dequantize_batch",
                     "cq_dequant_gemv_batch", "cq_fake_quantize_batch"}


def test_guard_helpers_detect_writes_past_either_end():
    torch = pytest.importorskip("torch")
    from tests import parity
    for dtype in (torch.uint8, torch.float16, torch.bfloat16, torch.float32):
        base, t = parity.guarded_empty((5, 7), dtype, "cpu")
        assert t.shape == (5, 7) and (t.data_ptr() - base.data_ptr()) == parity.GUARD_BYTES
        t.zero_()
        assert parity.guard_intact(base, t)
        flat = base.view(torch.uint8)
        n = t.numel() * t.element_size()
        flat[parity.GUARD_BYTES + n] = 0  # one byte past the end
        assert not parity.guard_intact(base, t)
        flat[parity.GUARD_BYTES + n] = parity.GUARD_FILL
        flat[parity.GUARD_BYTES - 1] = 0  # one byte before the start
        assert not parity.guard_intact(base, t)
