#!/usr/bin/env python
"""Benchmark: CQ quantise -> dequantise -> dequant-GEMV over a 7B-scale weight set on B200.

One step is one pass of the whole hot path over the synthetic Llama-shaped bf16 weight set
(32 layers of q/k/v/o 4096x4096, gate/up 11008x4096, down 4096x11008; 6,476,005,376
weights, N(0, 0.02^2), seed 3): 2-bit cq_quantize_batch over all 224 tensors,
cq_dequantize_batch of all of them back to bf16, and one cq_dequant_gemv_batch call with a
batch-1 product through every tensor.  Inputs are far larger than L2 (13 GB), so no flush is needed between steps.

  python bench.py [--gpus N] [--steps K] [--warmup W] [--impl cq|reference]

`value` is Gweights/s through the step (all ranks; weak scaling: each rank runs its own
replica of the set).  Per-op times, the same ops as one call per tensor, fake quantisation
(bf16 -> bf16 through the stored form), 4-bit quantise / dequantise and the GEMV-only
workload (the two MLP shapes over 48 distinct replicas, batch 1, 8 and 64) are reported in
`breakdown`.  `--impl reference` times the CPU oracle on a bounded sample instead.
"""
from __future__ import annotations

import argparse
import json
import math
import os
import statistics
import subprocess
import sys
import threading
import time

ROOT = os.path.dirname(os.path.abspath(__file__))
if ROOT not in sys.path:
    sys.path.insert(0, ROOT)

METRIC = "CQ quant/dequant Gweights/s & % HBM roofline; dequant-GEMV GB/s (1 B200)"
UNIT = "Gweights/s"
FALLBACK_HBM_GBS = 6650.0

BITS = 2
FIELD = {0: 2, 2: 2, 3: 3, 4: 4}


def bytes_per_weight_quant(bits: int, in_bytes: int = 2) -> float:
    """Algorithmic HBM bytes per weight: read the input, write b/8 index bytes + 2/128 norm."""
    return in_bytes + FIELD[bits] / 8 + 2 / 128


def bytes_per_weight_gemv(bits: int) -> float:
    return FIELD[bits] / 8 + 2 / 128


# ------------------------------------------------------------------------------------------
# distributed plumbing (also exercised by the CPU gloo tests)
# ------------------------------------------------------------------------------------------

def dist_env():
    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    return world, rank, local


def replica_tensor_offset(rank: int, n_tensors: int) -> int:
    """Each rank quantises its own replica of the weight set: tensor ids are offset per rank
    so replicas hold different data (no data is exchanged between ranks)."""
    return rank * n_tensors


def max_over_ranks(value: float, device=None) -> float:
    import torch
    import torch.distributed as dist
    if not (dist.is_available() and dist.is_initialized()):
        return value
    t = torch.tensor([value], dtype=torch.float64, device=device)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


def barrier():
    import torch.distributed as dist
    if dist.is_available() and dist.is_initialized():
        dist.barrier()


# ------------------------------------------------------------------------------------------
# clocks during the timed region
# ------------------------------------------------------------------------------------------

class ClockSampler:
    FIELDS = ("clocks.sm,clocks.max.sm,clocks_event_reasons.hw_slowdown,"
              "clocks_event_reasons.hw_thermal_slowdown,clocks_event_reasons.sw_thermal_slowdown,"
              "clocks_event_reasons.sw_power_cap")
    NAMES = ("hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap")

    def __init__(self, gpu_index: int):
        self.gpu = gpu_index
        self.proc = None
        self.lines = []
        self.first = 0

    def __enter__(self):
        try:
            self.proc = subprocess.Popen(
                ["nvidia-smi", f"--id={self.gpu}", f"--query-gpu={self.FIELDS}",
                 "--format=csv,noheader,nounits", "-lms", "50"],
                stdout=subprocess.PIPE, stderr=subprocess.DEVNULL, text=True)
            self.reader = threading.Thread(target=self._read, daemon=True)
            self.reader.start()
            # sampling is running before the timed region starts
            t0 = time.time()
            while not self.lines and time.time() - t0 < 3.0 and self.proc.poll() is None:
                time.sleep(0.01)
        except OSError:
            self.proc = None
        self.first = len(self.lines)
        return self

    def mark(self):
        """Only samples taken from now on count."""
        self.first = len(self.lines)

    def _read(self):
        for line in self.proc.stdout:
            self.lines.append(line.strip())

    def __exit__(self, *exc):
        if self.proc is not None:
            self.proc.terminate()
            try:
                self.proc.wait(timeout=5)
            except subprocess.TimeoutExpired:
                self.proc.kill()
            self.reader.join(timeout=5)

    def summary(self):
        sm, mx, reasons = [], [], set()
        for ln in self.lines[self.first:]:
            parts = [p.strip() for p in ln.split(",")]
            if len(parts) != 6:
                continue
            try:
                sm.append(float(parts[0]))
                mx.append(float(parts[1]))
            except ValueError:
                continue
            for name, val in zip(self.NAMES, parts[2:]):
                if val.lower().startswith("active"):
                    reasons.add(name)
        if not sm:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": ["unsampled"], "samples": 0}
        return {"sm_mhz": statistics.median(sm), "sm_max_mhz": max(mx),
                "reasons": sorted(reasons), "samples": len(sm)}


def nvsmi_id(device) -> str:
    """nvidia-smi --id for a torch device (its UUID, robust to CUDA_VISIBLE_DEVICES)."""
    import torch
    try:
        u = str(torch.cuda.get_device_properties(device).uuid)
        return u if u.startswith("GPU-") else "GPU-" + u
    except (AttributeError, RuntimeError):
        return str(device.index or 0)


def measured_peak_gbs():
    try:
        with open(os.path.join(ROOT, "MEASURED_PEAKS.json")) as f:
            d = json.load(f)
        return float(d["hbm_gbs"]), "measured"
    except (OSError, KeyError, ValueError):
        return FALLBACK_HBM_GBS, "fallback"


# ------------------------------------------------------------------------------------------
# the CUDA arm
# ------------------------------------------------------------------------------------------

class WeightSet:
    """One replica of the 7B-scale set in a single bf16 buffer, plus per-tensor views of the
    packed / norm / dequantised / GEMV buffers."""

    def __init__(self, workload, device, id_offset: int, bits: int):
        import torch
        import synth
        self.wl = workload
        self.bits = bits
        self.n = workload.numel
        self.groups = workload.groups
        blk = 16 * FIELD[bits]
        self.w = torch.empty(self.n, dtype=torch.bfloat16, device=device)
        self.packed = torch.empty(self.groups * blk, dtype=torch.uint8, device=device)
        self.norms = torch.empty(self.groups, dtype=torch.float16, device=device)
        self.out = torch.empty(self.n, dtype=torch.bfloat16, device=device)
        self.tensors = []
        off = goff = 0
        for t in workload.tensors:
            v = self.w[off:off + t.numel].view(t.rows, t.cols)
            synth.fill_normal_(v, workload.seed, t.tensor_id + id_offset, workload.sigma)
            G = -(-t.cols // 128)
            self.tensors.append(dict(
                t=t, w=v,
                packed=self.packed[goff * blk:(goff + t.groups) * blk].view(t.rows, G, blk),
                norms=self.norms[goff:goff + t.groups].view(t.rows, G),
                out=self.out[off:off + t.numel].view(t.rows, t.cols)))
            off += t.numel
            goff += t.groups
        # batch-1 activations, one per input width, and one output vector per tensor
        self.x = {}
        for c in sorted({t.cols for t in workload.tensors}):
            x = torch.empty((1, c), dtype=torch.bfloat16, device=device)
            synth.fill_normal_(x, workload.seed, 100000 + c + id_offset, 1.0)
            self.x[c] = x
        self.y = torch.empty(sum(t.rows for t in workload.tensors), dtype=torch.float32, device=device)
        yo = 0
        for d in self.tensors:
            d["y"] = self.y[yo:yo + d["t"].rows].view(1, -1)
            yo += d["t"].rows
        import hadamard_codebook_bit_b200 as cq
        self.ws = torch.empty(max(cq.gemv_workspace_bytes(c, 1) for c in self.x), dtype=torch.uint8,
                              device=device)
        # one workspace per tensor for the batched GEMV (its products run concurrently)
        wsb = [-(-cq.gemv_workspace_bytes(d["t"].cols, 1) // 256) * 256 for d in self.tensors]
        self.ws_all = torch.empty(sum(wsb), dtype=torch.uint8, device=device)
        off = 0
        for d, b in zip(self.tensors, wsb):
            d["ws"] = self.ws_all[off:off + b]
            off += b

    def quantize_all(self):
        """Every tensor of the set through one cq_quantize_batch call (the library's
        whole-model entry point)."""
        import hadamard_codebook_bit_b200 as cq
        cq.quantize_batch([d["w"] for d in self.tensors], self.bits,
                          outs=[(d["packed"], d["norms"]) for d in self.tensors])

    def dequantize_all(self):
        import hadamard_codebook_bit_b200 as cq
        cq.dequantize_batch([(d["packed"], d["norms"], d["t"].rows, d["t"].cols) for d in self.tensors],
                            self.bits, outs=[d["out"] for d in self.tensors])

    def fake_quantize_all(self):
        """W_hat = dequantize(quantize(W)) of every tensor through one cq_fake_quantize_batch
        call (the stored forms land in the packed / norms buffers)."""
        import hadamard_codebook_bit_b200 as cq
        cq.fake_quantize_batch([d["w"] for d in self.tensors], self.bits,
                               outs=[d["out"] for d in self.tensors],
                               stored=[(d["packed"], d["norms"]) for d in self.tensors])

    def quantize_each(self):
        """The same work as one cq_quantize call per tensor."""
        import hadamard_codebook_bit_b200 as cq
        for d in self.tensors:
            cq.quantize(d["w"], self.bits, out=(d["packed"], d["norms"]))

    def dequantize_each(self):
        import hadamard_codebook_bit_b200 as cq
        for d in self.tensors:
            t = d["t"]
            cq.dequantize(d["packed"], d["norms"], t.rows, t.cols, self.bits, out=d["out"])

    def gemv_all(self):
        """A batch-1 product through every tensor in one cq_dequant_gemv_batch call."""
        import hadamard_codebook_bit_b200 as cq
        cq.dequant_gemv_batch([(d["packed"], d["norms"], d["t"].rows, d["t"].cols, self.x[d["t"].cols])
                               for d in self.tensors], self.bits,
                              workspaces=[d["ws"] for d in self.tensors], ys=[d["y"] for d in self.tensors])

    def gemv_each(self):
        """The same products as one cq_dequant_gemv call per tensor."""
        import hadamard_codebook_bit_b200 as cq
        for d in self.tensors:
            t = d["t"]
            cq.dequant_gemv(d["packed"], d["norms"], t.rows, t.cols, self.bits, self.x[t.cols],
                            workspace=self.ws, y=d["y"])

    def launches_per_step(self) -> int:
        # batched quantise and dequantise (up to 128 tensors a launch), batched rotate-x + GEMV
        # (up to 256 products a launch pair)
        n = len(self.tensors)
        return 2 * -(-n // 128) + 2 * -(-n // 256)

    def capture(self, fns=None):
        """Capture each phase's calls in a CUDA graph (one replay per phase), so the host's
        per-call overhead stays off the GPU timeline."""
        import torch
        self.graphs = []
        for fn in (fns or (self.quantize_all, self.dequantize_all, self.gemv_all)):
            fn()  # first calls upload the default codebook (must precede capture)
            torch.cuda.synchronize()
            g = torch.cuda.CUDAGraph()
            with torch.cuda.graph(g):
                fn()
            self.graphs.append(g)
        return self.graphs

    def release(self):
        self.graphs = []


def time_phases(ws, steps: int, device):
    """Run `steps` steps, recording events between the phases; returns per-phase ms lists
    and the total (first start to last end) in ms."""
    import torch
    evs = []
    start = torch.cuda.Event(enable_timing=True)
    end = torch.cuda.Event(enable_timing=True)
    start.record()
    gq, gd, gg = ws.graphs
    for _ in range(steps):
        e = [torch.cuda.Event(enable_timing=True) for _ in range(4)]
        e[0].record()
        gq.replay()
        e[1].record()
        gd.replay()
        e[2].record()
        gg.replay()
        e[3].record()
        evs.append(e)
    end.record()
    torch.cuda.synchronize(device)
    q = [e[0].elapsed_time(e[1]) for e in evs]
    d = [e[1].elapsed_time(e[2]) for e in evs]
    g = [e[2].elapsed_time(e[3]) for e in evs]
    return q, d, g, start.elapsed_time(end)


def time_fn(fn, iters: int, device, warm: int = 2):
    import torch
    for _ in range(warm):
        fn()
    torch.cuda.synchronize(device)
    ts = []
    for _ in range(iters):
        a = torch.cuda.Event(enable_timing=True)
        b = torch.cuda.Event(enable_timing=True)
        a.record()
        fn()
        b.record()
        torch.cuda.synchronize(device)
        ts.append(a.elapsed_time(b))
    return ts


def gemv_replica_workload(device, peak):
    """The two MLP shapes, 2-bit, over 48 distinct quantised replicas (about 575 MB, far more
    than L2) called round-robin; per-call time = total / 48."""
    import torch
    import hadamard_codebook_bit_b200 as cq
    import synth
    from synth import workloads as wlm
    W = wlm.GEMV_7B
    reps = 48
    out = {}
    for ti, t in enumerate(W.tensors):
        w = torch.empty((t.rows, t.cols), dtype=torch.bfloat16, device=device)
        synth.fill_normal_(w, W.seed, t.tensor_id, W.sigma)
        pk, nm = cq.quantize(w, 2)
        del w
        pks = [pk.clone() for _ in range(reps)]
        nms = [nm.clone() for _ in range(reps)]
        for batch in tuple(W.extra["batches"]) + (64,):  # 64: a prefill-sized block of rows
            x = torch.empty((batch, t.cols), dtype=torch.bfloat16, device=device)
            synth.fill_normal_(x, W.seed, W.extra["x_ids"][ti], W.extra["x_sigma"])
            y = torch.empty((batch, t.rows), dtype=torch.float32, device=device)
            ws = torch.empty(cq.gemv_workspace_bytes(t.cols, batch), dtype=torch.uint8, device=device)

            def run():
                for i in range(reps):
                    cq.dequant_gemv(pks[i], nms[i], t.rows, t.cols, 2, x, workspace=ws, y=y)

            run()
            torch.cuda.synchronize(device)
            graph = torch.cuda.CUDAGraph()
            with torch.cuda.graph(graph):
                run()
            ts = time_fn(graph.replay, 5, device)
            del graph
            us = statistics.median(ts) / reps * 1000
            byts = t.groups * (32 + 2) + 2 * t.cols * batch + 4 * t.rows * batch
            gbs = byts / us / 1e3
            out[f"{t.rows}x{t.cols}_b{batch}"] = {"us_per_call": round(us, 3), "GB_s": round(gbs, 1),
                                                  "frac_hbm": round(gbs / peak, 4)}
        del pks, nms
    return out


def cpu_oracle_sample(target_s: float, threads: int = 0, max_rows: int = 4096):
    """Time the oracle on rows of layer 0's q tensor (4096 columns): 2-bit quantise,
    dequantise and a batch-1 GEMV, the same step as the GPU's.  The sample is the first
    `rows` rows, passed through the oracle repeatedly until about `target_s` seconds have
    elapsed.  Returns (Gweights/s, rows, passes, seconds, threads)."""
    import oracle
    import synth
    from synth import workloads as wlm
    W = wlm.LLAMA_7B
    t0 = W.tensors[0]
    cols = t0.cols
    x = synth.normal_host((1, cols), W.seed, 100000 + cols, 1.0, "bf16")
    nth = threads or oracle.default_threads()
    rows = 64
    w = synth.normal_host((rows, cols), W.seed, t0.tensor_id, W.sigma, "bf16")

    def one(wm, r):
        p, n = oracle.quantize(wm, BITS, nthreads=nth)
        oracle.dequantize(p, n, r, cols, BITS, nthreads=nth)
        oracle.dequant_gemv(p, n, r, cols, BITS, x, nthreads=nth)

    s = time.perf_counter()
    one(w, rows)
    dt = time.perf_counter() - s
    rows = int(max(64, min(max_rows, rows * 0.5 * target_s / max(dt, 1e-4))))
    w = synth.normal_host((rows, cols), W.seed, t0.tensor_id, W.sigma, "bf16")
    passes = 0
    s = time.perf_counter()
    while True:
        one(w, rows)
        passes += 1
        dt = time.perf_counter() - s
        if dt >= target_s:
            break
    return rows * cols * passes / dt / 1e9, rows, passes, dt, nth


def arm_config(world: int) -> dict:
    """The workload both arms report (the reference arm times a bounded sample of it, described
    in its cpu_baseline.sample)."""
    from synth import workloads as wlm
    return {"workload": "llama7b_bf16 weight set (6,476,005,376 weights, 224 tensors), 2-bit "
                        "quantize_batch + dequantize_batch(bf16) + dequant_gemv_batch (batch 1) over all "
                        "tensors, per step",
            "bits": BITS, "group_size": 128, "seed": wlm.LLAMA_7B.seed,
            "l2": "inputs (12.95 GB) larger than L2; no flush",
            "parallelism": f"replica per GPU x{world}"}


def run_cuda_arm(args):
    import torch
    world, rank, local = dist_env()
    device = torch.device(f"cuda:{local}")
    torch.cuda.set_device(device)
    if world > 1:
        import torch.distributed as dist
        from datetime import timedelta
        dist.init_process_group("nccl", timeout=timedelta(seconds=300), device_id=device)
    import hadamard_codebook_bit_b200 as cq
    from synth import workloads as wlm
    cq.lib()
    W = wlm.LLAMA_7B
    peak, peak_kind = measured_peak_gbs()

    ws = WeightSet(W, device, replica_tensor_offset(rank, len(W.tensors)), BITS)
    torch.cuda.synchronize(device)
    ws.capture()
    for _ in range(args.warmup):
        for g in ws.graphs:
            g.replay()
    torch.cuda.synchronize(device)
    barrier()
    torch.cuda.synchronize(device)
    with ClockSampler(nvsmi_id(device)) as clk:
        clk.mark()
        q_ms, d_ms, g_ms, total_ms = time_phases(ws, args.steps, device)
    torch.cuda.synchronize(device)
    barrier()
    total_ms = max_over_ranks(total_ms, device)
    clocks = clk.summary()

    n = W.numel
    ms_step = total_ms / args.steps
    value = world * n * args.steps / (total_ms / 1e3) / 1e9
    qm, dm, gm = (statistics.median(x) for x in (q_ms, d_ms, g_ms))
    qb = n * bytes_per_weight_quant(BITS)
    gb = n * bytes_per_weight_gemv(BITS)
    ops = {
        "quantize": {"ms": round(qm, 4), "Gweights_s": round(n / qm / 1e6, 1),
                     "GB_s": round(qb / qm / 1e6, 1), "frac_hbm": round(qb / qm / 1e6 / peak, 4)},
        "dequantize": {"ms": round(dm, 4), "Gweights_s": round(n / dm / 1e6, 1),
                       "GB_s": round(qb / dm / 1e6, 1), "frac_hbm": round(qb / dm / 1e6 / peak, 4)},
        "dequant_gemv": {"ms": round(gm, 4), "Gweights_s": round(n / gm / 1e6, 1),
                         "GB_s": round(gb / gm / 1e6, 1), "frac_hbm": round(gb / gm / 1e6 / peak, 4)},
    }
    dom = "quantize" if qm >= dm else "dequantize"
    dom_ms = max(qm, dm)
    achieved = qb / dom_ms / 1e6
    traffic = load_traffic(dom, n)

    breakdown = {"ops_2bit": ops}
    if not args.quick:
        # the same two phases as one call per tensor (224 launches each)
        ge, gd, gg = ws.capture((ws.quantize_each, ws.dequantize_each, ws.gemv_each))
        qe = statistics.median(time_fn(ge.replay, 5, device))
        de = statistics.median(time_fn(gd.replay, 5, device))
        gme = statistics.median(time_fn(gg.replay, 5, device))
        ws.release()
        breakdown["ops_2bit_one_call_per_tensor"] = {
            "quantize": {"ms": round(qe, 4), "GB_s": round(qb / qe / 1e6, 1), "frac_hbm": round(qb / qe / 1e6 / peak, 4)},
            "dequantize": {"ms": round(de, 4), "GB_s": round(qb / de / 1e6, 1), "frac_hbm": round(qb / de / 1e6 / peak, 4)},
            "dequant_gemv": {"ms": round(gme, 4), "GB_s": round(gb / gme / 1e6, 1), "frac_hbm": round(gb / gme / 1e6 / peak, 4)}}
        ws.release()
        # fake quantisation (the pages' cq_quantize output): bf16 W -> bf16 W_hat, two launches
        # per 128 tensors through the stored form; its own roofline is the fused minimum of
        # 4 B/weight (read W, write W_hat), the two steps move 2 x 2.265625 B/weight
        (gf,) = ws.capture((ws.fake_quantize_all,))
        fq = statistics.median(time_fn(gf.replay, 5, device))
        ws.release()
        fb = n * 4.0
        breakdown["fake_quantize_2bit"] = {
            "ms": round(fq, 4), "Gweights_s": round(n / fq / 1e6, 1),
            "GB_s": round(fb / fq / 1e6, 1), "frac_hbm": round(fb / fq / 1e6 / peak, 4),
            "algorithmic_bytes_per_weight": 4.0, "moved_bytes_per_weight": 2 * bytes_per_weight_quant(BITS)}
        del ws
        torch.cuda.empty_cache()
        ws4 = WeightSet(W, device, replica_tensor_offset(rank, len(W.tensors)), 4)
        g4q, g4d, _ = ws4.capture()
        q4 = statistics.median(time_fn(g4q.replay, 5, device))
        d4 = statistics.median(time_fn(g4d.replay, 5, device))
        ws4.release()
        qb4 = n * bytes_per_weight_quant(4)
        breakdown["ops_4bit"] = {
            "quantize": {"ms": round(q4, 4), "Gweights_s": round(n / q4 / 1e6, 1),
                         "GB_s": round(qb4 / q4 / 1e6, 1), "frac_hbm": round(qb4 / q4 / 1e6 / peak, 4)},
            "dequantize": {"ms": round(d4, 4), "Gweights_s": round(n / d4 / 1e6, 1),
                           "GB_s": round(qb4 / d4 / 1e6, 1), "frac_hbm": round(qb4 / d4 / 1e6 / peak, 4)}}
        del ws4
        torch.cuda.empty_cache()
        breakdown["gemv_7b_mlp_48_replicas"] = gemv_replica_workload(device, peak)
        ws = WeightSet(W, device, replica_tensor_offset(rank, len(W.tensors)), BITS)
        ws.capture()

    e2e = None
    if not args.no_e2e:
        e2e = run_e2e(ws, args, device, world)

    cpu = None
    if rank == 0 and world == 1 and not args.no_cpu_baseline:
        v, rows, passes, dt, nth = cpu_oracle_sample(args.cpu_seconds)
        cpu = {"value": round(v, 6), "unit": UNIT, "cores": nth, "kind": "oracle",
               "sample": f"first {rows} rows (x4096, bf16) of tensor l0.q, {passes} passes of "
                         f"2-bit quantise + dequantise + batch-1 GEMV, {dt:.1f} s"}

    ws.release()
    if rank == 0:
        line = {
            "metric": METRIC, "value": round(value, 3), "unit": UNIT, "n_gpus": world,
            "steps": args.steps, "warmup": args.warmup, "ms_per_step": round(ms_step, 4),
            "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "bf16",
            "data": "synthetic",
            "config": arm_config(world),
            "roofline": {"bound": "hbm", "kernel": f"cq_{dom}", "achieved": round(achieved, 1),
                         "peak": peak, "peak_kind": peak_kind, "unit": "GB/s",
                         "frac": round(achieved / peak, 4), "traffic": traffic},
            "breakdown": breakdown,
            "cpu_baseline": cpu,
            "e2e": e2e,
            "clocks": clocks,
            "gpu_launches": ws.launches_per_step() * args.steps,
        }
        print(json.dumps(line), flush=True)
    if world > 1:
        import torch.distributed as dist
        dist.destroy_process_group()


def load_traffic(kernel: str, n_weights: int):
    """DRAM bytes per launch-unit from the committed ncu summary, scaled to this launch, or
    None if the summary is missing or was taken on a different source of that kernel (its
    .cu file and the headers it includes)."""
    path = os.path.join(ROOT, "profiles", "traffic.json")
    try:
        with open(path) as f:
            d = json.load(f)
        ent = d[kernel]
        from hadamard_codebook_bit_b200 import build as b
        if ent.get("source_hash") != b.source_hash(ent.get("sources")):
            return None
        return round(ent["dram_bytes_per_weight"] * n_weights)
    except (OSError, KeyError, ValueError, AttributeError, FileNotFoundError):
        return None


def run_e2e(ws, args, device, world):
    """Same step through the public API with the inputs in pinned HOST memory: each step
    copies the bf16 weights and the activations host->device, runs quantise / dequantise /
    GEMV, and reads packed + norms + dequantised weights + y back to pinned host memory."""
    import torch
    steps = max(1, min(args.steps, 3))
    w_h = torch.empty_like(ws.w, device="cpu").pin_memory()
    w_h.copy_(ws.w)
    x_h = {c: x.cpu().pin_memory() for c, x in ws.x.items()}
    packed_h = torch.empty_like(ws.packed, device="cpu").pin_memory()
    norms_h = torch.empty_like(ws.norms, device="cpu").pin_memory()
    out_h = torch.empty_like(ws.out, device="cpu").pin_memory()
    y_h = torch.empty_like(ws.y, device="cpu").pin_memory()
    h2d = ws.w.numel() * 2 + sum(x.numel() * 2 for x in ws.x.values())
    d2h = ws.packed.numel() + ws.norms.numel() * 2 + ws.out.numel() * 2 + ws.y.numel() * 4

    def step():
        ws.w.copy_(w_h, non_blocking=True)
        for c, x in ws.x.items():
            x.copy_(x_h[c], non_blocking=True)
        for g in ws.graphs:
            g.replay()
        packed_h.copy_(ws.packed, non_blocking=True)
        norms_h.copy_(ws.norms, non_blocking=True)
        out_h.copy_(ws.out, non_blocking=True)
        y_h.copy_(ws.y, non_blocking=True)

    step()
    torch.cuda.synchronize(device)
    barrier()
    a = torch.cuda.Event(enable_timing=True)
    b = torch.cuda.Event(enable_timing=True)
    a.record()
    for _ in range(steps):
        step()
    b.record()
    torch.cuda.synchronize(device)
    barrier()
    ms = max_over_ranks(a.elapsed_time(b), device)
    return {"value": round(world * ws.n * steps / (ms / 1e3) / 1e9, 3), "unit": UNIT,
            "h2d_bytes_per_step": h2d, "d2h_bytes_per_step": d2h, "steps": steps,
            "ms_per_step": round(ms / steps, 2)}


# ------------------------------------------------------------------------------------------
# the reference arm: the CPU oracle, as it stands, on a bounded sample
# ------------------------------------------------------------------------------------------

def run_reference_arm(args):
    world, rank, _ = dist_env()
    if rank != 0:
        return
    import oracle
    oracle.build()
    per_step = max(1.0, min(8.0, 150.0 / max(1, args.steps + args.warmup)))
    vals = []
    rows = None
    nth = oracle.default_threads()
    passes = 0
    for i in range(args.warmup + args.steps):
        v, rows, passes, dt, nth = cpu_oracle_sample(per_step)
        if i >= args.warmup:
            vals.append(v)
    value = statistics.median(vals)
    sample = (f"first {rows} rows (x4096, bf16) of tensor l0.q per step, {passes} passes of "
              f"2-bit quantise + dequantise + batch-1 GEMV (~{per_step:.0f} s per step)")
    from synth import workloads as wlm
    line = {
        "impl": "reference", "metric": METRIC, "value": round(value, 6), "unit": UNIT,
        "n_gpus": world, "steps": args.steps, "warmup": args.warmup,
        "ms_per_step": round(rows * 4096 * passes / (value * 1e9) * 1e3, 2),
        "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "f64",
        "data": "synthetic",
        "config": arm_config(world),
        "cpu_baseline": {"value": round(value, 6), "unit": UNIT, "cores": nth, "kind": "oracle",
                         "sample": sample},
        "e2e": {"value": round(value, 6), "unit": UNIT, "h2d_bytes_per_step": 0,
                "d2h_bytes_per_step": 0},
    }
    print(json.dumps(line), flush=True)


def run_ncu_case(args):
    """Small fixed launches for a detailed ncu capture, in the form the bench step uses them:
    eight 4096x4096 bf16 tensors (256 MiB, larger than L2) through cq_quantize_batch,
    cq_dequantize_batch and a batch-1 cq_dequant_gemv_batch, then one 11008x4096 2-bit
    cq_dequant_gemv at batch 1 and 8.  Each call runs 1 + 3 times (the first is a warm-up)."""
    import torch
    import hadamard_codebook_bit_b200 as cq
    import synth
    device = torch.device("cuda:0")
    n_t, rows, cols, bits = 8, 4096, 4096, args.ncu_bits
    ws = []
    for k in range(n_t):
        w = torch.empty((rows, cols), dtype=torch.bfloat16, device=device)
        synth.fill_normal_(w, 3, k, 0.02)
        ws.append(w)
    outs = [cq.empty_packed(rows, cols, bits, device) for _ in range(n_t)]
    deq = [torch.empty_like(w) for w in ws]
    for _ in range(4):
        cq.quantize_batch(ws, bits, outs=outs)
    items = [(pk, nm, rows, cols) for pk, nm in outs]
    for _ in range(4):
        cq.dequantize_batch(items, bits, outs=deq)
    x = torch.empty((1, cols), dtype=torch.bfloat16, device=device)
    synth.fill_normal_(x, 4, 100, 1.0)
    if bits in (0, 2):
        g_items = [(pk, nm, rows, cols, x) for pk, nm in outs]
        for _ in range(4):
            cq.dequant_gemv_batch(g_items, bits)
    g_rows, g_cols = 11008, 4096
    wg = torch.empty((g_rows, g_cols), dtype=torch.bfloat16, device=device)
    synth.fill_normal_(wg, 4, 0, 0.02)
    pk, nm = cq.quantize(wg, 2)
    for batch in (1, 8):
        xb = torch.empty((batch, g_cols), dtype=torch.bfloat16, device=device)
        synth.fill_normal_(xb, 4, 100, 1.0)
        for _ in range(4):
            cq.dequant_gemv(pk, nm, g_rows, g_cols, 2, xb)
    torch.cuda.synchronize(device)
    print(json.dumps({"ncu_case": "done", "tensors": n_t, "rows": rows, "cols": cols, "bits": bits}))


def main():
    ap = argparse.ArgumentParser(description=__doc__, formatter_class=argparse.RawDescriptionHelpFormatter)
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=20)
    ap.add_argument("--warmup", type=int, default=3)
    ap.add_argument("--impl", choices=["cq", "reference"], default="cq")
    ap.add_argument("--quick", action="store_true", help="skip the 4-bit and GEMV-replica extras")
    ap.add_argument("--no-e2e", action="store_true")
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--cpu-seconds", type=float, default=12.0)
    ap.add_argument("--ncu-case", action="store_true",
                    help="run the small fixed launches used for detailed ncu captures and exit")
    ap.add_argument("--ncu-bits", type=int, default=2)
    args = ap.parse_args()
    if args.ncu_case:
        run_ncu_case(args)
        return
    if args.warmup < 3:
        ap.error("--warmup must be >= 3")
    if args.impl == "reference":
        run_reference_arm(args)
    else:
        run_cuda_arm(args)


if __name__ == "__main__":
    main()
