"""The bench's multi-rank plumbing on CPU: two gloo ranks, no GPU."""
import os
import socket

import pytest
import torch
import torch.distributed as dist
import torch.multiprocessing as mp

import bench


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _worker(rank, world, port, q):
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port), RANK=str(rank),
                      WORLD_SIZE=str(world), LOCAL_RANK=str(rank))
    dist.init_process_group("gloo", rank=rank, world_size=world)
    try:
        w, r, local = bench.dist_env()
        assert (w, r, local) == (world, rank, rank)
        bench.barrier()
        m = bench.max_over_ranks(10.0 + rank * 5.0)  # the slowest rank decides
        off = bench.replica_tensor_offset(rank, 224)
        q.put((rank, m, off))
    finally:
        dist.destroy_process_group()


def test_two_gloo_ranks_time_max_and_disjoint_replicas():
    world, port = 2, _free_port()
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    procs = [ctx.Process(target=_worker, args=(r, world, port, q)) for r in range(world)]
    for p in procs:
        p.start()
    for p in procs:
        p.join(timeout=120)
        assert p.exitcode == 0
    res = sorted(q.get(timeout=5) for _ in range(world))
    assert [m for _, m, _ in res] == [15.0, 15.0]
    offs = [o for _, _, o in res]
    assert offs == [0, 224]  # tensor ids of the two replicas do not overlap


def test_single_process_helpers_without_process_group():
    assert bench.max_over_ranks(3.5) == 3.5
    bench.barrier()
    assert bench.bytes_per_weight_quant(2) == 2.265625
    assert bench.bytes_per_weight_quant(4) == 2.515625
    assert bench.bytes_per_weight_quant(3) == 2.390625
    assert bench.bytes_per_weight_gemv(2) == 0.265625


def test_clock_sampler_parses_nvidia_smi_lines():
    c = bench.ClockSampler(0)
    c.lines = ["1965, 1965, Not Active, Not Active, Not Active, Active",
               "1800, 1965, Not Active, Not Active, Not Active, Not Active",
               "garbage"]
    s = c.summary()
    assert s["sm_mhz"] == 1882.5 and s["sm_max_mhz"] == 1965 and s["reasons"] == ["sw_power_cap"]


def test_load_traffic_scales_per_weight_and_checks_the_source_hash(monkeypatch):
    import json
    from hadamard_codebook_bit_b200 import build as cq_build
    with open(os.path.join(os.path.dirname(bench.__file__), "profiles", "traffic.json")) as f:
        table = json.load(f)
    n = 6_476_005_376
    for kernel in ("quantize", "dequantize", "dequant_gemv"):
        ent = table[kernel]
        assert abs(ent["dram_bytes_per_weight"] - (ent["dram_read_bytes"] + ent["dram_write_bytes"]) / 134217728) < 1e-4
        monkeypatch.setattr(cq_build, "source_hash", lambda files=None, h=ent["source_hash"]: h)
        assert bench.load_traffic(kernel, n) == round(ent["dram_bytes_per_weight"] * n)
    monkeypatch.setattr(cq_build, "source_hash", lambda files=None: "0" * 16)  # kernel changed since capture
    assert bench.load_traffic("dequantize", n) is None
    assert bench.load_traffic("no_such_kernel", n) is None


def test_arm_config_names_the_workload():
    c1, c4 = bench.arm_config(1), bench.arm_config(4)
    assert "6,476,005,376 weights" in c1["workload"] and c1["bits"] == 2 and c1["group_size"] == 128
    assert c1["parallelism"] != c4["parallelism"] and "4" in c4["parallelism"]


def test_source_hash_of_named_files():
    from hadamard_codebook_bit_b200 import build as cq_build
    a = cq_build.source_hash(["cq_gemv.cu", "cq.h"])
    assert a == cq_build.source_hash(["cq.h", "cq_gemv.cu"]) and a != cq_build.source_hash(["cq_gemv.cu"])
    assert len(cq_build.source_hash()) == 16
    with pytest.raises(FileNotFoundError):
        cq_build.source_hash(["no_such_file.cu"])
