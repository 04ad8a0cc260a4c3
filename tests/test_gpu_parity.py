"""GPU parity: the CUDA path (through the C ABI) against the fp64 CPU oracle.

Every comparison feeds both sides the same bytes: inputs made on the device are copied
back for the oracle, and dequantise / GEMV parity is measured on the packed arrays the GPU
produced.  Tolerances are in tests/parity.py.
"""
import math

import numpy as np
import pytest

torch = pytest.importorskip("torch")

import hadamard_codebook_bit_b200 as cq  # noqa: E402
import synth  # noqa: E402
from synth import workloads as wl  # noqa: E402
from tests import parity  # noqa: E402

pytestmark = pytest.mark.gpu

DEV = "cuda:0"


@pytest.fixture(scope="module", autouse=True)
def _gpu():
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    from hadamard_codebook_bit_b200 import build
    build.build()
    synth.build()
    torch.cuda.init()


@pytest.fixture(scope="module")
def ora(oracle_lib):
    return oracle_lib


def to_np(t):
    """Device tensor -> numpy with the oracle's conventions (bf16/fp16 as uint16 bits)."""
    t = t.detach().contiguous().cpu()
    if t.dtype in (torch.bfloat16, torch.float16):
        return t.view(torch.int16).numpy().view(np.uint16)
    return t.numpy()


def dev_tensor(rows, cols, dtype, seed, tid, sigma):
    t = torch.empty((rows, cols), dtype=dtype, device=DEV)
    synth.fill_normal_(t, seed, tid, sigma)
    return t


def roundtrip_check(ora, w_dev, bits, what, codebook=None, out_dtypes=("f32", "bf16")):
    """Quantise on the GPU and check against the oracle; then dequantise the GPU's packed
    arrays on both sides.  Returns (packed, norms, w_np, flips)."""
    rows, cols = w_dev.shape
    cb_dev = None if codebook is None else torch.tensor(codebook, dtype=torch.float32, device=DEV)
    cb = cq.codebook(bits) if codebook is None else np.asarray(codebook, np.float32)
    packed, norms = cq.quantize(w_dev, bits, codebook=cb_dev)
    torch.cuda.synchronize()
    w_np = to_np(w_dev)
    o_packed, o_norms, u = ora.quantize(w_np, bits, codebook_=cb, want_u=True)
    g_packed, g_norms = to_np(packed), to_np(norms)
    flips = parity.check_indices(g_packed, o_packed, u, bits, cb, what)
    w64 = w_np.astype(np.float64) if w_np.dtype != np.uint16 else parity.bf16_to_f64(w_np).reshape(rows, cols)
    parity.check_norms(g_norms, o_norms, parity.group_norms(w64, cols), what)
    ref = ora.dequantize(g_packed, g_norms, rows, cols, bits, codebook_=cb)
    if "f32" in out_dtypes:
        out = cq.dequantize(packed, norms, rows, cols, bits, codebook=cb_dev, out_dtype=torch.float32)
        parity.check_dequant_f32(to_np(out), ref, cols, what + " f32")
    if "bf16" in out_dtypes:
        out = cq.dequantize(packed, norms, rows, cols, bits, codebook=cb_dev, out_dtype=torch.bfloat16)
        parity.check_dequant_bf16(to_np(out), ref, cols, what + " bf16")
    return g_packed, g_norms, w64, flips


# ------------------------------------------------------------------------------------------
# the synthetic generator itself
# ------------------------------------------------------------------------------------------

@pytest.mark.parametrize("dtype", ["f32", "bf16"])
def test_device_generator_matches_host(dtype):
    tdt = torch.float32 if dtype == "f32" else torch.bfloat16
    for n, off in [(1, 0), (7, 3), (100003, 0), (4096, 12345)]:
        t = torch.empty(n, dtype=tdt, device=DEV)
        synth.fill_normal_(t, 9, 4, 0.02, offset=off)
        host = synth.normal_host((n,), 9, 4, 0.02, dtype, offset=off)
        assert np.array_equal(to_np(t), host)


# ------------------------------------------------------------------------------------------
# the five workloads
# ------------------------------------------------------------------------------------------

def test_small_fp32_matrix(ora):
    w = wl.SMALL_FP32
    t = w.tensors[0]
    host = synth.normal_host((t.rows, t.cols), w.seed, t.tensor_id, w.sigma, "f32")
    w_dev = torch.from_numpy(host).to(DEV)
    packed, norms, w64, _ = roundtrip_check(ora, w_dev, 2, "small_fp32")
    assert packed.size == cq.packed_bytes(t.rows, t.cols, 2) == 32768
    assert norms.size * 2 == cq.norm_bytes(t.rows, t.cols) == 2048
    deq = ora.dequantize(packed, norms, t.rows, t.cols, 2)
    rel = float(np.sum((w64 - deq) ** 2) / np.sum(w64 ** 2))
    assert 0.10 < rel < 0.13  # expected ~0.116 for a group-normalised Gaussian source


@pytest.mark.parametrize("bits", [0, 2, 3, 4])
def test_outlier_sweep(ora, bits):
    w_np = wl.outlier_sweep_host()
    w_dev = torch.from_numpy(w_np).to(DEV)
    roundtrip_check(ora, w_dev, bits, f"outlier bits={bits}", out_dtypes=("f32",))


def test_needle_45m_set(ora):
    w = wl.NEEDLE_45M
    total_packed = total_norm = 0
    for t in w.tensors:
        w_dev = dev_tensor(t.rows, t.cols, torch.bfloat16, w.seed, t.tensor_id, w.sigma)
        out = ("f32", "bf16") if t.name in ("head", "l0.k") else ("bf16",)
        packed, norms, _, _ = roundtrip_check(ora, w_dev, 2, f"needle {t.name}", out_dtypes=out)
        total_packed += packed.size
        total_norm += norms.size * 2
    assert (total_packed, total_norm) == (11206656, 700416)


@pytest.mark.parametrize("bits", [2, 4])
def test_llama7b_sampled(ora, bits):
    """Full 7B-scale set on the device, quantised tensor by tensor exactly as the benchmark
    does; sampled groups from every tensor checked against the oracle, and every group's
    norm checked against torch's fp32 norm of the input."""
    w = wl.LLAMA_7B
    rng = np.random.default_rng(bits)
    cb = cq.codebook(bits)
    per_tensor = 256
    ins, outs_p, outs_n = [], [], []
    for t in w.tensors:
        w_dev = dev_tensor(t.rows, t.cols, torch.bfloat16, w.seed, t.tensor_id, w.sigma)
        packed, norms = cq.quantize(w_dev, bits)
        # property at full size: stored norm = fp16(||group||) up to fp16 rounding
        ref = w_dev.float().view(-1, 128).norm(dim=1)
        got = norms.float().view(-1)
        assert torch.all((got - ref).abs() <= ref * 2.0 ** -10 + 1e-12), t.name
        gidx = torch.from_numpy(rng.choice(t.groups, per_tensor, replace=False)).to(DEV)
        ins.append(to_np(w_dev.view(-1, 128)[gidx]))
        outs_p.append(to_np(packed.view(t.groups, -1)[gidx]))
        outs_n.append(to_np(norms.view(-1)[gidx]))
        del w_dev, packed, norms
    w_np = np.concatenate(ins)
    g_packed, g_norms = np.concatenate(outs_p), np.concatenate(outs_n)
    o_packed, o_norms, u = ora.quantize(w_np, bits, codebook_=cb, want_u=True)
    parity.check_indices(g_packed, o_packed, u, bits, cb, "llama7b")
    parity.check_norms(g_norms, o_norms, parity.group_norms(parity.bf16_to_f64(w_np).reshape(-1, 128), 128))
    # dequantise the sampled groups on both sides from the GPU's packed arrays
    rows = w_np.shape[0]
    pk = torch.from_numpy(g_packed).to(DEV)
    nm = torch.from_numpy(g_norms.view(np.float16)).to(DEV)
    deq = cq.dequantize(pk, nm, rows, 128, bits, out_dtype=torch.bfloat16)
    parity.check_dequant_bf16(to_np(deq), ora.dequantize(g_packed, g_norms, rows, 128, bits), 128, "llama7b")


@pytest.mark.parametrize("ti", [0, 1])
@pytest.mark.parametrize("batch", [1, 8])
def test_gemv_7b_shapes(ora, ti, batch):
    w = wl.GEMV_7B
    t = w.tensors[ti]
    w_dev = dev_tensor(t.rows, t.cols, torch.bfloat16, w.seed, t.tensor_id, w.sigma)
    packed, norms = cq.quantize(w_dev, 2)
    x = torch.empty((batch, t.cols), dtype=torch.bfloat16, device=DEV)
    synth.fill_normal_(x, w.seed, w.extra["x_ids"][ti], w.extra["x_sigma"])
    y = cq.dequant_gemv(packed, norms, t.rows, t.cols, 2, x)
    torch.cuda.synchronize()
    y_ref = ora.dequant_gemv(to_np(packed), to_np(norms), t.rows, t.cols, 2, to_np(x))
    parity.check_gemv(to_np(y), y_ref, f"gemv {t.name} b={batch}")


# ------------------------------------------------------------------------------------------
# edge cases
# ------------------------------------------------------------------------------------------

@pytest.mark.parametrize("cols", [1, 7, 8, 100, 127, 128, 129, 255, 1000, 1001, 4100])
@pytest.mark.parametrize("dtype", [torch.float32, torch.bfloat16])
def test_ragged_columns(ora, cols, dtype):
    rows = 37
    w_dev = dev_tensor(rows, cols, dtype, 11, cols, 0.5)
    for bits in (0, 2, 3, 4):
        roundtrip_check(ora, w_dev, bits, f"cols={cols} {dtype} bits={bits}")


@pytest.mark.parametrize("bits", [0, 2, 3, 4])
@pytest.mark.parametrize("cols,batch", [(1, 1), (130, 3), (1000, 8), (4096, 2)])
def test_gemv_all_bits_and_ragged(ora, bits, cols, batch):
    rows = 45
    w_dev = dev_tensor(rows, cols, torch.bfloat16, 12, cols, 0.02)
    packed, norms = cq.quantize(w_dev, bits)
    x = torch.empty((batch, cols), dtype=torch.bfloat16, device=DEV)
    synth.fill_normal_(x, 12, 1000 + cols, 1.0)
    y = cq.dequant_gemv(packed, norms, rows, cols, bits, x)
    y_ref = ora.dequant_gemv(to_np(packed), to_np(norms), rows, cols, bits, to_np(x))
    parity.check_gemv(to_np(y), y_ref, f"gemv bits={bits} cols={cols}")


@pytest.mark.parametrize("bits", [0, 2, 3, 4])
@pytest.mark.parametrize("batch", [9, 16, 33, 64])
def test_gemv_prefill_batches(ora, bits, batch):
    """Batches above 8 activation rows (up to 64) run as blocks of 8 in one launch pair."""
    rows, cols = 70, 1000
    w_dev = dev_tensor(rows, cols, torch.bfloat16, 15, batch + bits, 0.02)
    packed, norms = cq.quantize(w_dev, bits)
    x = torch.empty((batch, cols), dtype=torch.bfloat16, device=DEV)
    synth.fill_normal_(x, 15, 2000 + batch, 1.0)
    y = cq.dequant_gemv(packed, norms, rows, cols, bits, x)
    y_ref = ora.dequant_gemv(to_np(packed), to_np(norms), rows, cols, bits, to_np(x))
    parity.check_gemv(to_np(y), y_ref, f"gemv bits={bits} batch={batch}")
    # the batched entry point with mixed batch sizes gives the same products
    x8 = x[:8].contiguous()
    ys = cq.dequant_gemv_batch([(packed, norms, rows, cols, x), (packed, norms, rows, cols, x8)], bits)
    torch.cuda.synchronize()
    parity.check_gemv(to_np(ys[0]), y_ref, f"gemv batch-call bits={bits} batch={batch}")
    parity.check_gemv(to_np(ys[1]), y_ref[:8], f"gemv batch-call bits={bits} batch=8")


def test_zero_and_spike_groups(ora):
    w = torch.zeros((6, 384), dtype=torch.float32, device=DEV)
    w[1, 5] = 0.37
    w[2, 128 + 77] = -2.5
    w[3, :] = 1.0  # constant rows rotate onto one component
    w[4, 256:] = -0.001
    for bits in (0, 2, 3, 4):
        roundtrip_check(ora, w, bits, f"special bits={bits}")


def test_custom_codebook(ora):
    cb = np.array([-0.2, -0.05, 0.01, 0.15], np.float32)  # asymmetric, caller supplied
    w_dev = dev_tensor(64, 640, torch.bfloat16, 13, 0, 0.02)
    roundtrip_check(ora, w_dev, 2, "custom codebook", codebook=cb)


@pytest.mark.parametrize("bits", [3, 4])
def test_custom_codebook_wide_levels(ora, bits):
    """A caller codebook with evenly spread levels: the bucket-table search handles it."""
    cb = np.linspace(-0.25, 0.21, 1 << bits).astype(np.float32)
    w_dev = dev_tensor(96, 1024, torch.bfloat16, 30, bits, 0.02)
    roundtrip_check(ora, w_dev, bits, f"wide codebook {bits}-bit", codebook=cb)


@pytest.mark.parametrize("bits", [3, 4])
def test_custom_codebook_crowded_levels(ora, bits):
    """Two midpoints closer than a bucket: the quantiser falls back to the select tree."""
    cb = np.linspace(-0.25, 0.21, 1 << bits).astype(np.float32)
    cb[3] = cb[2] + 1e-4  # levels 2, 3 nearly equal -> midpoints 1|2 and 2|3 share a bucket
    cb[4] = cb[3] + 2e-4
    w_dev = dev_tensor(96, 1024, torch.bfloat16, 31, bits, 0.02)
    roundtrip_check(ora, w_dev, bits, f"crowded codebook {bits}-bit", codebook=cb)


def test_unused_ternary_code_decodes_as_top_level(ora):
    packed = torch.full((3, 2, 32), 0xFF, dtype=torch.uint8, device=DEV)  # every code = 3
    norms = torch.full((3, 2), 1.5, dtype=torch.float16, device=DEV)
    out = cq.dequantize(packed, norms, 3, 256, 0, out_dtype=torch.float32)
    ref = ora.dequantize(to_np(packed), to_np(norms), 3, 256, 0)
    parity.check_dequant_f32(to_np(out), ref, 256, "ternary code 3")


def test_empty_inputs():
    w = torch.empty((0, 128), dtype=torch.bfloat16, device=DEV)
    packed, norms = cq.quantize(w, 2)
    assert packed.numel() == 0 and norms.numel() == 0
    y = torch.full((2, 5), 7.0, device=DEV)
    x = torch.empty((2, 0), dtype=torch.bfloat16, device=DEV)
    p = torch.empty((5, 0, 32), dtype=torch.uint8, device=DEV)
    n = torch.empty((5, 0), dtype=torch.float16, device=DEV)
    cq.dequant_gemv(p, n, 5, 0, 2, x, workspace=torch.empty(16, dtype=torch.uint8, device=DEV), y=y)
    torch.cuda.synchronize()
    assert torch.all(y == 0)


def test_deterministic_and_stream_ordered(ora):
    w_dev = dev_tensor(300, 4096, torch.bfloat16, 14, 0, 0.02)
    s = torch.cuda.Stream()
    with torch.cuda.stream(s):
        a = cq.quantize(w_dev, 3)
        b = cq.quantize(w_dev, 3)
    s.synchronize()
    assert torch.equal(a[0], b[0]) and torch.equal(a[1], b[1])
    c = cq.quantize(w_dev, 3)
    assert torch.equal(a[0], c[0]) and torch.equal(a[1], c[1])


def test_more_than_2g_elements_sampled(ora):
    """A single tensor of 2^31 + 2^20 bf16 elements (offsets beyond int32)."""
    rows, cols = 16640, 129088  # 2,147,624,...: cols % 128 == 64 -> padded groups too
    assert rows * cols > 2 ** 31
    w_dev = dev_tensor(rows, cols, torch.bfloat16, 15, 0, 0.02)
    packed, norms = cq.quantize(w_dev, 2)
    out = cq.dequantize(packed, norms, rows, cols, 2, out_dtype=torch.bfloat16)
    rng = np.random.default_rng(0)
    sel = np.sort(rng.choice(rows, 6, replace=False))
    sel[-1] = rows - 1
    w_np = to_np(w_dev[torch.from_numpy(sel).to(DEV)])
    o_packed, o_norms, u = ora.quantize(w_np, 2, want_u=True)
    g_packed = to_np(packed[torch.from_numpy(sel).to(DEV)])
    g_norms = to_np(norms[torch.from_numpy(sel).to(DEV)])
    parity.check_indices(g_packed, o_packed, u, 2, cq.codebook(2), "2G")
    parity.check_norms(g_norms, o_norms, parity.group_norms(parity.bf16_to_f64(w_np), cols))
    ref = ora.dequantize(g_packed, g_norms, len(sel), cols, 2)
    parity.check_dequant_bf16(to_np(out[torch.from_numpy(sel).to(DEV)]), ref, cols, "2G deq")


# shapes for the batched calls: flat, row-tiled, CUDA-core (cols % 8 != 0), tiny and empty
BATCH_SHAPES = [(256, 512), (37, 1000), (64, 100), (1, 128), (300, 4096), (5, 8), (0, 128),
                (129, 256), (3, 11008)]


def batch_tensor(rows, cols, dtype, seed, tid, sigma):
    if rows * cols == 0:
        return torch.empty((rows, cols), dtype=dtype, device=DEV)
    return dev_tensor(rows, cols, dtype, seed, tid, sigma)


@pytest.mark.parametrize("bits", [0, 2, 4])
def test_quantize_batch_equals_single_calls(ora, bits):
    """One cq_quantize_batch over assorted shapes returns exactly the bytes of one cq_quantize
    per tensor; the single calls are the ones checked against the oracle elsewhere, and one
    batched job is also checked against the oracle here."""
    ws = [batch_tensor(r, c, torch.bfloat16, 21, k, 0.02) for k, (r, c) in enumerate(BATCH_SHAPES)]
    got = cq.quantize_batch(ws, bits)
    for w, (pb, nb) in zip(ws, got):
        ps, ns = cq.quantize(w, bits)
        assert torch.equal(pb, ps) and torch.equal(nb.view(torch.int16), ns.view(torch.int16))
    w_np = to_np(ws[1])
    o_packed, o_norms, u = ora.quantize(w_np, bits, want_u=True)
    parity.check_indices(to_np(got[1][0]), o_packed, u, bits, cq.codebook(bits), "batch job 1")
    parity.check_norms(to_np(got[1][1]), o_norms, parity.group_norms(parity.bf16_to_f64(w_np), 1000))


def test_quantize_batch_many_jobs_and_fp32():
    """More jobs than one launch carries (chunked launches), and an fp32 batch (CUDA-core
    path for every job)."""
    shapes = [(3 + (k % 5), 128 * (1 + k % 3)) for k in range(150)]
    ws = [dev_tensor(r, c, torch.bfloat16, 22, k, 0.02) for k, (r, c) in enumerate(shapes)]
    got = cq.quantize_batch(ws, 2)
    for w, (pb, nb) in zip(ws, got):
        ps, ns = cq.quantize(w, 2)
        assert torch.equal(pb, ps) and torch.equal(nb.view(torch.int16), ns.view(torch.int16))
    wf = [batch_tensor(r, c, torch.float32, 23, k, 1.0) for k, (r, c) in enumerate(BATCH_SHAPES)]
    got = cq.quantize_batch(wf, 3)
    for w, (pb, nb) in zip(wf, got):
        ps, ns = cq.quantize(w, 3)
        assert torch.equal(pb, ps) and torch.equal(nb.view(torch.int16), ns.view(torch.int16))


@pytest.mark.parametrize("bits", [0, 2, 3, 4])
@pytest.mark.parametrize("out_dtype", [torch.bfloat16, torch.float32])
def test_dequantize_batch_equals_single_calls(bits, out_dtype):
    ws = [batch_tensor(r, c, torch.bfloat16, 24, k, 0.02) for k, (r, c) in enumerate(BATCH_SHAPES)]
    q = cq.quantize_batch(ws, bits)
    items = [(pk, nm, r, c) for (pk, nm), (r, c) in zip(q, BATCH_SHAPES)]
    got = cq.dequantize_batch(items, bits, out_dtype=out_dtype)
    for (pk, nm, r, c), ob in zip(items, got):
        os_ = cq.dequantize(pk, nm, r, c, bits, out_dtype=out_dtype)
        assert ob.shape == (r, c) and torch.equal(ob.view(-1).view(torch.int16 if out_dtype == torch.bfloat16 else torch.int32),
                                                 os_.view(-1).view(torch.int16 if out_dtype == torch.bfloat16 else torch.int32))


def test_dequantize_batch_many_jobs():
    shapes = [(2 + (k % 7), 128 * (1 + k % 4)) for k in range(140)]
    ws = [dev_tensor(r, c, torch.bfloat16, 25, k, 0.02) for k, (r, c) in enumerate(shapes)]
    q = cq.quantize_batch(ws, 2)
    items = [(pk, nm, r, c) for (pk, nm), (r, c) in zip(q, shapes)]
    got = cq.dequantize_batch(items, 2)
    for (pk, nm, r, c), ob in zip(items, got):
        assert torch.equal(ob.view(torch.int16), cq.dequantize(pk, nm, r, c, 2).view(torch.int16))


# ------------------------------------------------------------------------------------------
# fake quantisation: W_hat = dequantize(quantize(W)) in one call
# ------------------------------------------------------------------------------------------

def _int_view(t):
    return t.view(torch.int16) if t.element_size() == 2 else t.view(torch.int32)


def fake_check(ora, w_dev, bits, out_dtype, what):
    """cq_fake_quantize against (1) the library's own two-step result, bit for bit, and
    (2) the oracle's fake quantisation of the same input, group by group where the stored
    forms agree, and the oracle's dequantisation of the GPU's stored form where an index sits
    inside the boundary band (check_indices bounds those)."""
    rows, cols = w_dev.shape
    stored = cq.empty_packed(rows, cols, bits, w_dev.device)
    out = cq.fake_quantize(w_dev, bits, out_dtype=out_dtype, stored=stored)
    ps, ns = cq.quantize(w_dev, bits)
    assert torch.equal(stored[0], ps) and torch.equal(stored[1].view(torch.int16), ns.view(torch.int16))
    two_step = cq.dequantize(ps, ns, rows, cols, bits, out_dtype=out_dtype)
    assert out.dtype == out_dtype and torch.equal(_int_view(out), _int_view(two_step))
    w_np = to_np(w_dev)
    o_packed, o_norms, u = ora.quantize(w_np, bits, want_u=True)
    g_packed, g_norms = to_np(ps), to_np(ns)
    parity.check_indices(g_packed, o_packed, u, bits, cq.codebook(bits), what)
    w64 = w_np.astype(np.float64) if w_np.dtype != np.uint16 else parity.bf16_to_f64(w_np).reshape(rows, cols)
    parity.check_norms(g_norms, o_norms, parity.group_norms(w64, cols), what)
    ref = ora.fake_quantize(w_np, bits)
    same = np.all(g_packed == o_packed, axis=-1) & (g_norms == o_norms)  # [rows, G]
    if not same.all():
        alt = ora.dequantize(g_packed, g_norms, rows, cols, bits)
        cmask = np.repeat(same, 128, axis=1)[:, :cols]
        ref = np.where(cmask, ref, alt)
    if out_dtype == torch.float32:
        parity.check_dequant_f32(to_np(out), ref, cols, what)
    else:
        parity.check_dequant_bf16(to_np(out), ref, cols, what)
    return int((~same).sum())


@pytest.mark.parametrize("bits", [0, 2, 3, 4])
@pytest.mark.parametrize("cols", [128, 1000, 4096])
def test_fake_quantize_matches_oracle(ora, bits, cols):
    w_dev = dev_tensor(70, cols, torch.bfloat16, 40, cols + bits, 0.02)
    fake_check(ora, w_dev, bits, torch.bfloat16, f"fake bf16 bits={bits} cols={cols}")
    fake_check(ora, w_dev, bits, torch.float32, f"fake bf16->f32 bits={bits} cols={cols}")


@pytest.mark.parametrize("cols", [1, 129, 4100])
def test_fake_quantize_fp32_ragged_and_special(ora, cols):
    w_dev = dev_tensor(33, cols, torch.float32, 41, cols, 1.0)
    w_dev[3, :] = 0.0
    w_dev[4, :] = 0.0
    w_dev[4, cols // 2] = -2.5  # spike group
    for bits in (0, 2, 4):
        fake_check(ora, w_dev, bits, torch.float32, f"fake f32 bits={bits} cols={cols}")


def test_fake_quantize_in_place_and_batch():
    """out = w (in place) gives the out-of-place result; the batched call gives the single
    calls' bytes, in place too, over assorted (and empty) shapes."""
    w = dev_tensor(300, 4096, torch.bfloat16, 42, 0, 0.02)
    want = cq.fake_quantize(w, 2)
    w2 = w.clone()
    got = cq.fake_quantize(w2, 2, out=w2)
    assert got.data_ptr() == w2.data_ptr() and torch.equal(_int_view(w2), _int_view(want))
    ws = [batch_tensor(r, c, torch.bfloat16, 43, k, 0.02) for k, (r, c) in enumerate(BATCH_SHAPES)]
    singles = [cq.fake_quantize(x, 4) for x in ws]
    outs = cq.fake_quantize_batch(ws, 4)
    for a, b in zip(outs, singles):
        assert a.shape == b.shape and torch.equal(_int_view(a), _int_view(b))
    copies = [x.clone() for x in ws]
    cq.fake_quantize_batch(copies, 4, outs=copies)
    for a, b in zip(copies, singles):
        assert torch.equal(_int_view(a), _int_view(b))
    many = [dev_tensor(2 + k % 5, 128 * (1 + k % 3), torch.float32, 44, k, 1.0) for k in range(150)]
    outs = cq.fake_quantize_batch(many, 3, out_dtype=torch.bfloat16)
    for k in (0, 127, 128, 149):
        assert torch.equal(_int_view(outs[k]), _int_view(cq.fake_quantize(many[k], 3, out_dtype=torch.bfloat16)))


@pytest.mark.parametrize("bits", [0, 2, 4])
def test_gemv_batch_matches_oracle(ora, bits):
    """cq_dequant_gemv_batch over assorted products (ragged, several batch sizes, empty rows,
    empty inner dimension) against the oracle, and repeatable bit for bit."""
    shapes = [(37, 1000, 3), (256, 4096, 1), (64, 128, 8), (1, 129, 2), (0, 256, 1), (5, 0, 2),
              (300, 11008, 1)]
    items, refs = [], []
    for k, (r, c, b) in enumerate(shapes):
        w = batch_tensor(r, c, torch.bfloat16, 26, k, 0.02)
        pk, nm = cq.quantize(w, bits)
        x = batch_tensor(b, c, torch.bfloat16, 27, k, 1.0)
        items.append((pk, nm, r, c, x))
    ys = cq.dequant_gemv_batch(items, bits)
    ys2 = cq.dequant_gemv_batch(items, bits)
    torch.cuda.synchronize()
    for (pk, nm, r, c, x), y, y2 in zip(items, ys, ys2):
        assert y.shape == (x.shape[0], r) and torch.equal(y, y2)
        if r == 0:
            continue
        if c == 0:
            assert torch.all(y == 0)
            continue
        ref = ora.dequant_gemv(to_np(pk), to_np(nm), r, c, bits, to_np(x))
        parity.check_gemv(to_np(y), ref, f"gemv batch {r}x{c} b={x.shape[0]}")


def test_gemv_batch_many_jobs(ora):
    """More products than one launch pair carries."""
    items = []
    for k in range(260):
        r, c = 3 + k % 5, 128 * (1 + k % 3)
        pk, nm = cq.quantize(dev_tensor(r, c, torch.bfloat16, 28, k, 0.02), 2)
        items.append((pk, nm, r, c, dev_tensor(1, c, torch.bfloat16, 29, k, 1.0)))
    ys = cq.dequant_gemv_batch(items, 2)
    torch.cuda.synchronize()
    for k in (0, 1, 128, 255, 256, 259):
        pk, nm, r, c, x = items[k]
        ref = ora.dequant_gemv(to_np(pk), to_np(nm), r, c, 2, to_np(x))
        parity.check_gemv(to_np(ys[k]), ref, f"gemv batch job {k}")


# ------------------------------------------------------------------------------------------
# guard bytes: no kernel writes outside its output buffers (memory checkers are not available
# here, so every output sits between margins of a fixed byte pattern that must survive)
# ------------------------------------------------------------------------------------------

@pytest.mark.parametrize("bits", [0, 2, 3, 4])
@pytest.mark.parametrize("rows,cols,dtype", [(37, 1000, torch.bfloat16), (5, 129, torch.float32),
                                             (130, 4096, torch.bfloat16), (1, 8, torch.bfloat16),
                                             (3, 11008, torch.bfloat16), (9, 100, torch.bfloat16)])
def test_outputs_stay_inside_their_buffers(bits, rows, cols, dtype):
    w = dev_tensor(rows, cols, dtype, 50, cols + bits, 0.02)
    ref_p, ref_n = cq.quantize(w, bits)
    G = -(-cols // 128)
    bp, gp = parity.guarded_empty((rows, G, 16 * parity.field_bits(bits)), torch.uint8, DEV)
    bn, gn = parity.guarded_empty((rows, G), torch.float16, DEV)
    cq.quantize(w, bits, out=(gp, gn))
    torch.cuda.synchronize()
    assert parity.guard_intact(bp, gp) and parity.guard_intact(bn, gn)
    assert torch.equal(gp, ref_p) and torch.equal(gn.view(torch.int16), ref_n.view(torch.int16))
    for out_dtype in (torch.bfloat16, torch.float32):
        ref_o = cq.dequantize(ref_p, ref_n, rows, cols, bits, out_dtype=out_dtype)
        bo, go = parity.guarded_empty((rows, cols), out_dtype, DEV)
        cq.dequantize(ref_p, ref_n, rows, cols, bits, out=go)
        bf, gf = parity.guarded_empty((rows, cols), out_dtype, DEV)
        cq.fake_quantize(w, bits, out=gf)
        torch.cuda.synchronize()
        assert parity.guard_intact(bo, go) and parity.guard_intact(bf, gf)
        assert torch.equal(_int_view(go), _int_view(ref_o)) and torch.equal(_int_view(gf), _int_view(ref_o))
    for batch in (1, 8, 20):
        x = dev_tensor(batch, cols, torch.bfloat16, 51, cols + batch, 1.0)
        ref_y = cq.dequant_gemv(ref_p, ref_n, rows, cols, bits, x)
        bw, gw = parity.guarded_empty((cq.gemv_workspace_bytes(cols, batch),), torch.uint8, DEV)
        by, gy = parity.guarded_empty((batch, rows), torch.float32, DEV)
        cq.dequant_gemv(ref_p, ref_n, rows, cols, bits, x, workspace=gw, y=gy)
        torch.cuda.synchronize()
        assert parity.guard_intact(bw, gw) and parity.guard_intact(by, gy)
        assert torch.equal(gy, ref_y)


@pytest.mark.parametrize("bits", [0, 2, 4])
def test_batched_outputs_stay_inside_their_buffers(bits):
    ws = [batch_tensor(r, c, torch.bfloat16, 52, k, 0.02) for k, (r, c) in enumerate(BATCH_SHAPES)]
    fb = parity.field_bits(bits)
    gq = [(parity.guarded_empty((r, -(-c // 128), 16 * fb), torch.uint8, DEV),
           parity.guarded_empty((r, -(-c // 128)), torch.float16, DEV)) for r, c in BATCH_SHAPES]
    cq.quantize_batch(ws, bits, outs=[(p[1], n[1]) for p, n in gq])
    go = [parity.guarded_empty((r, c), torch.bfloat16, DEV) for r, c in BATCH_SHAPES]
    cq.dequantize_batch([(p[1], n[1], r, c) for (p, n), (r, c) in zip(gq, BATCH_SHAPES)], bits,
                        outs=[o[1] for o in go])
    gf = [parity.guarded_empty((r, c), torch.float32, DEV) for r, c in BATCH_SHAPES]
    cq.fake_quantize_batch(ws, bits, outs=[f[1] for f in gf])
    items, gy, gw = [], [], []
    for k, ((p, n), (r, c)) in enumerate(zip(gq, BATCH_SHAPES)):
        b = 1 + k % 3
        items.append((p[1], n[1], r, c, batch_tensor(b, c, torch.bfloat16, 53, k, 1.0)))
        gy.append(parity.guarded_empty((b, r), torch.float32, DEV))
        gw.append(parity.guarded_empty((max(cq.gemv_workspace_bytes(c, b), 16),), torch.uint8, DEV))
    cq.dequant_gemv_batch(items, bits, workspaces=[w_[1] for w_ in gw], ys=[y[1] for y in gy])
    torch.cuda.synchronize()
    for (p, n), o, f, y, w_, x, (r, c) in zip(gq, go, gf, gy, gw, ws, BATCH_SHAPES):
        for base, t in (p, n, o, f, y, w_):
            assert parity.guard_intact(base, t), (r, c)
        sp, sn = cq.quantize(x, bits)
        assert torch.equal(p[1], sp) and torch.equal(n[1].view(torch.int16), sn.view(torch.int16))
        assert torch.equal(o[1].view(torch.int16), cq.dequantize(sp, sn, r, c, bits).view(torch.int16))
        assert torch.equal(f[1].view(torch.int32),
                           cq.dequantize(sp, sn, r, c, bits, out_dtype=torch.float32).view(torch.int32))


def test_zz_no_kernel_wait_gave_up():
    """Every bounded wait inside the tensor-core kernels completed during this module."""
    assert cq.device_status() == 0
