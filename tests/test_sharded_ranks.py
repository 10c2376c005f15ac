"""The KV-sharded request on CPU: the shard plan, and two gloo ranks that each attend over
their own rows (the oracle stands in for the GPU), all-gather the partials and merge them by
log-sum-exp, which must give the oracle's attention over the whole request."""

import os
import socket

import numpy as np
import pytest
import torch
import torch.distributed as dist
import torch.multiprocessing as mp

import oracle
from mla_latent_kv_28_b200 import sharded


def test_shard_ranges_cover_in_order_on_tile_boundaries():
    for L in (0, 1, 63, 64, 65, 1000, 4096, 131072):
        for world in (1, 2, 3, 4, 8):
            r = sharded.shard_ranges(L, world)
            assert len(r) == world and r[0][0] == 0 and r[-1][1] == L
            for (a, b), (c, d) in zip(r, r[1:]):
                assert b == c and a <= b
            for a, b in r[:-1]:
                assert (a % 64 == 0 or a == L) and (b % 64 == 0 or b == L)
            tiles = [(b - a + 63) // 64 for a, b in r]
            assert max(tiles) - min(tiles) <= 1
    assert sharded.local_lengths([100, 10], 1, 2) == [36, 0]


def _lse_merge(lat_all, lse_all):
    m = np.max(lse_all, axis=0)
    w = np.where(np.isneginf(lse_all), 0.0, np.exp(lse_all - np.where(np.isneginf(m), 0.0, m)))
    den = w.sum(axis=0)
    lat = np.einsum("pbh,pbhc->bhc", w, lat_all) / np.where(den > 0, den, 1.0)[..., None]
    return lat, np.where(den > 0, m + np.log(np.where(den > 0, den, 1.0)), -np.inf)


def _rank(rank, world, port, result):
    os.environ["MASTER_ADDR"] = "127.0.0.1"
    os.environ["MASTER_PORT"] = str(port)
    dist.init_process_group("gloo", rank=rank, world_size=world)
    try:
        rng = np.random.default_rng(80)
        B, H, lens = 3, 4, [300, 64, 10]
        cache = rng.standard_normal((B, max(lens), 576))
        q = rng.standard_normal((B, H, 576)) * 0.3
        local = np.zeros((B, max(lens), 576))
        mine = []
        for b, L in enumerate(lens):
            a, e = sharded.shard_ranges(L, world)[rank]
            local[b, : e - a] = cache[b, a:e]
            mine.append(e - a)
        lat, lse = oracle.latent_attention(q, local, mine, 0.07)
        lat_all, lse_all = sharded.gather_partials(torch.from_numpy(lat), torch.from_numpy(lse))
        got_lat, got_lse = _lse_merge(lat_all.numpy(), lse_all.numpy())
        ref_lat, ref_lse = oracle.latent_attention(q, cache, lens, 0.07)
        result[rank] = float(max(np.max(np.abs(got_lat - ref_lat)), np.max(np.abs(got_lse - ref_lse))))
    finally:
        dist.destroy_process_group()


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


@pytest.mark.parametrize("world", [2, 3])
def test_gloo_ranks_gather_and_merge_to_the_whole_request(world):
    ctx = mp.get_context("spawn")
    mgr = ctx.Manager()
    result = mgr.dict()
    port = _free_port()
    procs = [ctx.Process(target=_rank, args=(r, world, port, result)) for r in range(world)]
    for p in procs:
        p.start()
    for p in procs:
        p.join(120)
        assert p.exitcode == 0
    assert len(result) == world
    for r in range(world):
        assert result[r] < 1e-10, (r, result[r])
