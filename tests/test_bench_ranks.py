"""The multi-rank plumbing of bench.py on CPU: two gloo ranks, as torchrun would start them.

Every rank runs its own replica of the workload (sequences are independent, no data-path
collective); the step time is the max over ranks and the throughput counts all ranks."""
import os
import socket

import pytest
import torch
import torch.multiprocessing as mp

import bench
from mla_latent_kv_28_b200 import workloads as wl


def _free_port() -> int:
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _rank_main(rank: int, world: int, port: int, out):
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port), RANK=str(rank),
                      WORLD_SIZE=str(world), LOCAL_RANK=str(rank))
    r, w, local = bench.dist_env()
    assert (r, w, local) == (rank, world, rank)
    dist = bench.init_dist(w, local, "gloo")
    try:
        bench.barrier(w, local, cuda=False)
        # each rank's own step time; every rank must see the slowest one
        ms = 1.0 + rank
        out[rank] = bench.max_over_ranks(ms, w, torch.device("cpu"))
        # replicas differ between ranks
        seqs = wl.config_workload("tiny_h16_l256", seed=bench.replica_seed(rank)).q_c
        out[world + rank] = float(seqs.float().sum())
        bench.barrier(w, local, cuda=False)
    finally:
        dist.destroy_process_group()


def test_two_gloo_ranks():
    world = 2
    ctx = mp.get_context("spawn")
    out = ctx.Array("d", 2 * world)
    port = _free_port()
    procs = [ctx.Process(target=_rank_main, args=(r, world, port, out)) for r in range(world)]
    for p in procs:
        p.start()
    for p in procs:
        p.join(timeout=120)
        assert p.exitcode == 0
    assert out[0] == out[1] == 2.0                      # max over ranks, seen by both
    assert out[2] != out[3]                             # different replica per rank


def test_job_throughput_counts_all_ranks():
    # 4 ranks x 32 sequences, the slowest rank at 2 ms per step: 64,000 tokens/s
    assert bench.job_tokens_per_s(4, 32, 2.0) == pytest.approx(64000.0)
    assert bench.job_tokens_per_s(1, 32, 2.0) == pytest.approx(16000.0)


def test_single_rank_needs_no_process_group():
    assert bench.max_over_ranks(3.5, 1, torch.device("cpu")) == 3.5
    bench.barrier(1, 0, cuda=False)  # a no-op without a process group


def test_committed_decode_profile_parses():
    """The ncu summary bench.py reads roofline.traffic from has its hash and byte count lines."""
    import bench
    path = os.path.join(os.path.dirname(os.path.dirname(os.path.abspath(__file__))), "profiles",
                        "decode_attn_v2_b32_l4096.txt")
    vals = {}
    with open(path) as f:
        for line in f:
            if ":" in line and not line.startswith("#"):
                k, v = line.split(":", 1)
                vals[k.strip()] = v.strip()
    assert len(vals["kernel_sources_sha"]) == 16
    assert float(vals["dram_bytes_per_launch"]) > float(vals["algorithmic_bytes_per_launch"]) * 0.9
    # while the kernel sources are the profiled ones, bench reports the traffic
    if vals["kernel_sources_sha"] == bench.kernel_sources_sha():
        assert bench.profiled_traffic("v2_b32_l4096") == float(vals["dram_bytes_per_launch"])
