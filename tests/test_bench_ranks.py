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


@pytest.mark.parametrize("workload", ["ragged_paged_b64", "v2_b32_l4096"])
def test_committed_decode_profile_parses(workload):
    """The ncu summaries bench.py reads roofline.traffic from have their hash and byte count
    lines (the headline workload's is taken on the current kernel sources)."""
    import bench
    path = os.path.join(os.path.dirname(os.path.dirname(os.path.abspath(__file__))), "profiles",
                        f"decode_attn_{workload}.txt")
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
        assert bench.profiled_traffic(workload) == float(vals["dram_bytes_per_launch"])
    if workload == bench.DEFAULT_WORKLOAD:
        assert vals["kernel_sources_sha"] == bench.kernel_sources_sha()


def _run_bench(*args, timeout=600):
    import subprocess
    import sys
    root = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
    env = {k: v for k, v in os.environ.items()
           if k not in ("RANK", "WORLD_SIZE", "LOCAL_RANK", "MASTER_ADDR", "MASTER_PORT")}
    env["CUDA_VISIBLE_DEVICES"] = ""
    return subprocess.run([sys.executable, os.path.join(root, "bench.py"), *args],
                          capture_output=True, text=True, timeout=timeout, cwd=root, env=env)


def test_gpus_n_without_torchrun_starts_n_ranks():
    """`--gpus 2` outside torchrun relaunches itself as two ranks: the reference arm then runs
    on rank 0 alone (the other rank exits 0 without work) and reports n_gpus 2."""
    import json
    r = _run_bench("--gpus", "2", "--impl", "reference", "--workload", "tiny_h16_l256",
                   "--steps", "2", "--warmup", "3")
    assert r.returncode == 0, r.stderr[-2000:]
    lines = [json.loads(x) for x in r.stdout.splitlines() if x.startswith("{")]
    assert len(lines) == 1 and lines[0]["n_gpus"] == 2 and lines[0]["impl"] == "reference"


def test_gpus_n_never_measures_fewer_gpus():
    """Without GPUs, `--gpus 2` fails loudly (each rank needs a GPU) instead of printing a
    one-GPU line; a WORLD_SIZE that disagrees with --gpus is refused."""
    r = _run_bench("--gpus", "2", "--workload", "tiny_h16_l256", "--steps", "2", "--warmup", "3",
                   "--no-cpu-baseline")
    assert r.returncode != 0
    assert '"n_gpus": 1' not in r.stdout
    import subprocess
    import sys
    root = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
    env = dict(os.environ, WORLD_SIZE="1", RANK="0", LOCAL_RANK="0", CUDA_VISIBLE_DEVICES="")
    r2 = subprocess.run([sys.executable, os.path.join(root, "bench.py"), "--gpus", "2"],
                        capture_output=True, text=True, timeout=300, cwd=root, env=env)
    assert r2.returncode == 2 and "WORLD_SIZE" in r2.stderr


def test_reference_arm_and_cpu_baseline_time_the_same_units():
    """Both CPU figures come from OracleSample: the same units, cut per head group."""
    w = wl.config_workload("tiny_h16_l256")
    s = bench.OracleSample(w)
    assert abs(s.run(0) - bench.HEADS_PER_UNIT / w.n_heads) < 1e-12
    tps, units, secs, desc = bench.oracle_tokens_per_s(w, budget_s=0.5)
    assert tps > 0 and units >= 1 and "heads of one sequence" in desc
