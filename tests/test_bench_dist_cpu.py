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
