"""The allocation-free GEMV entry point (collected last on purpose).

cq_dequant_gemv_static serves callers that cannot allocate device memory (for example
while a stream is being captured into a CUDA graph, or inside a host framework that owns
the allocator): it takes its scratch from an array inside the library instead of a caller
workspace.  Its output must match cq_dequant_gemv's on the same inputs, call after call.
"""
import ctypes

import numpy as np
import pytest

torch = pytest.importorskip("torch")

import hadamard_codebook_bit_b200 as cq  # noqa: E402
import synth  # noqa: E402
from tests import parity  # noqa: E402

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module", autouse=True)
def _gpu():
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    from hadamard_codebook_bit_b200 import build
    build.build()
    synth.build()


def _static_call(packed, norms, rows, cols, bits, x, y, stream):
    """Raw C-ABI call of cq_dequant_gemv_static (no workspace argument)."""
    return cq.lib().cq_dequant_gemv_static(
        ctypes.c_void_p(packed.data_ptr()), ctypes.c_void_p(norms.data_ptr()), rows, cols, bits,
        128, None, ctypes.c_void_p(x.data_ptr()), x.shape[0], ctypes.c_void_p(y.data_ptr()),
        ctypes.c_void_p(stream))


@pytest.mark.parametrize("rows,cols,bits,batch", [(11008, 4096, 2, 1), (4096, 11008, 2, 8),
                                                  (300, 1000, 3, 3), (64, 32768, 4, 2),
                                                  (300, 1000, 2, 20)])
def test_static_scratch_gemv_matches_workspace_gemv_twice(rows, cols, bits, batch):
    dev = torch.device("cuda:0")
    w = torch.empty((rows, cols), dtype=torch.bfloat16, device=dev)
    synth.fill_normal_(w, 21, cols, 0.02)
    packed, norms = cq.quantize(w, bits)
    x = torch.empty((batch, cols), dtype=torch.bfloat16, device=dev)
    synth.fill_normal_(x, 21, 7 + cols, 1.0)
    ref = cq.dequant_gemv(packed, norms, rows, cols, bits, x)  # caller-workspace entry point
    stream = torch.cuda.current_stream(dev).cuda_stream
    outs = []
    for _ in range(2):  # two calls in a row share (and rewrite) the static scratch
        y = torch.full((batch, rows), float("nan"), dtype=torch.float32, device=dev)
        assert _static_call(packed, norms, rows, cols, bits, x, y, stream) == 0
        outs.append(y)
    torch.cuda.synchronize()
    r = ref.cpu().numpy().astype(np.float64)
    # Up to 8 activation rows both entry points launch the same kernels with the same split:
    # identical bits.  Above 8 the static one runs its blocks one launch pair at a time, so
    # its split-K (chosen per launch) and hence the fp32 summation order may differ.
    same_bits = batch <= 8
    for y in outs:
        parity.check_gemv(y.cpu().numpy(), r, "static scratch")
        assert torch.equal(y, outs[0])
        if same_bits:
            assert torch.equal(y, ref)
    y3 = cq.dequant_gemv_static(packed, norms, rows, cols, bits, x)
    torch.cuda.synchronize()
    assert torch.equal(y3, outs[0])


def test_static_scratch_rejects_columns_beyond_its_size():
    dev = torch.device("cuda:0")
    cols = 32768 + 1
    packed = torch.zeros((1, 257, 32), dtype=torch.uint8, device=dev)
    norms = torch.zeros((1, 257), dtype=torch.float16, device=dev)
    x = torch.zeros((1, cols), dtype=torch.bfloat16, device=dev)
    y = torch.zeros((1, 1), dtype=torch.float32, device=dev)
    assert _static_call(packed, norms, 1, cols, 2, x, y, 0) == 5  # CQ_ERR_WORKSPACE
    with pytest.raises(cq.CQError):
        cq.dequant_gemv_static(packed, norms, 1, cols, 2, x, y=y)
