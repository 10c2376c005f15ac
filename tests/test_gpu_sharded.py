"""A long request whose cache rows are split over several GPUs, with the ranks emulated on one
GPU: each shard's partial (mla_decode_attn_partial over the rows it holds, query rotated at the
global position) and the log-sum-exp merge (mla_merge_partials) must give the oracle's
attention over the whole request. A one-rank NCCL group runs the ShardedDecode plumbing."""

import os
import socket

import numpy as np
import pytest
import torch
import torch.distributed as dist

import oracle
from mla_latent_kv_28_b200 import binding, sharded
from mla_latent_kv_28_b200 import workloads as wl
from tests._parity import assert_close, f64, to_np, workload_np

pytestmark = pytest.mark.gpu

DEV = "cuda:0"


def _local_cache(cache, lens, rank, world):
    """This rank's rows of each sequence, as a contiguous cache [B, max local, 576]."""
    rng = [sharded.shard_ranges(int(L), world)[rank] for L in lens]
    n = max(1, max(e - a for a, e in rng))
    local = torch.full((cache.shape[0], n, 576), float("nan"), dtype=torch.bfloat16, device=DEV)
    for b, (a, e) in enumerate(rng):
        local[b, : e - a] = cache[b, a:e]
    return local, torch.tensor([e - a for a, e in rng], dtype=torch.int32, device=DEV)


@pytest.mark.parametrize("world", [2, 4])
def test_shard_partials_merge_to_the_whole_request(world):
    w = wl.make_workload(2, 128, [20000, 333], seed=81)
    g = w.to(DEV)
    a = workload_np(w)
    full = binding.MlaDecode(128, 2, w.max_kv_len)
    # the oracle's absorbed query (global positions) in bf16 feeds both sides, so no oracle
    # input comes from the CUDA path
    q_ref = oracle.absorb_query(a["q_c"], a["q_r"], a["w_uk"], a["kv_lens"], w.rope_base)
    q_bf = torch.from_numpy(q_ref).to(torch.float32).to(torch.bfloat16)
    q_abs = q_bf.to(DEV)
    lat_parts, lse_parts = [], []
    for r in range(world):
        local, lens = _local_cache(g.cache, w.kv_lens.tolist(), r, world)
        h = binding.MlaDecode(128, 2, local.shape[1])
        lat, lse = h.decode_attn_partial(q_abs, local, lens)
        h.check_device_errors()
        lat_parts.append(lat)
        lse_parts.append(lse)
    latent, lse = full.merge_partials(torch.stack(lat_parts), torch.stack(lse_parts))
    full.check_device_errors()
    ref_lat, ref_lse = oracle.latent_attention(to_np(q_bf), a["cache"], a["kv_lens"],
                                               oracle.default_scale())
    assert_close(f64(latent), ref_lat, f"{world} shards merged: latent")
    assert_close(lse.cpu().numpy(), ref_lse, f"{world} shards merged: lse")
    # a shard with no rows of sequence 1 (333 rows = 6 tiles over 4 ranks leaves none empty,
    # but over 8 it would): its lse is -inf and the merge ignores it
    assert torch.isfinite(torch.stack(lse_parts)[:, 0]).all()


def test_empty_shard_is_ignored():
    w = wl.make_workload(1, 32, [100], seed=82)
    g = w.to(DEV)
    qa = wl.draw_q_abs(1, 32, seed=83).to(DEV)
    h = binding.MlaDecode(32, 1, 100)
    lat, lse = h.decode_attn_partial(qa, g.cache, g.kv_lens)
    empty_lat, empty_lse = h.decode_attn_partial(qa, g.cache, torch.zeros(1, dtype=torch.int32, device=DEV))
    assert torch.isneginf(empty_lse).all() and (empty_lat == 0).all()
    merged, mlse = h.merge_partials(torch.stack([empty_lat, lat]), torch.stack([empty_lse, lse]))
    direct, dlse = h.decode_attn(qa, g.cache, g.kv_lens)
    h.check_device_errors()
    # one real part: the merge only rounds the fp32 partial to bf16, as the direct call does
    assert torch.equal(merged, direct)
    assert torch.allclose(mlse, dlse, rtol=0, atol=1e-5)


def test_sharded_decode_over_a_one_rank_nccl_group():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        port = s.getsockname()[1]
    os.environ["MASTER_ADDR"] = "127.0.0.1"
    os.environ["MASTER_PORT"] = str(port)
    dist.init_process_group("nccl", rank=0, world_size=1)
    try:
        w = wl.make_workload(2, 64, [700, 50], seed=84)
        g = w.to(DEV)
        a = workload_np(w)
        h = binding.MlaDecode(64, 2, w.max_kv_len)
        sd = sharded.ShardedDecode(h)
        out = sd.step(g.q_c, g.q_r, g.w_uk, g.w_uv, g.kv_lens, g.cache, g.kv_lens)
        h.check_device_errors()
        ref = oracle.mla_decode_nonabsorbed(a["q_c"], a["q_r"], a["w_uk"], a["w_uv"], a["cache"],
                                            a["kv_lens"], oracle.default_scale(), w.rope_base)
        assert_close(f64(out), ref, "ShardedDecode, one rank: head outputs")
    finally:
        dist.destroy_process_group()


def test_partial_with_several_new_tokens_is_refused():
    h = binding.MlaDecode(16, 1, 64, q_len=2)
    qa = torch.zeros((1, 2, 16, 576), dtype=torch.bfloat16, device=DEV)
    cache = torch.zeros((1, 64, 576), dtype=torch.bfloat16, device=DEV)
    with pytest.raises(binding.MlaError, match="UNSUPPORTED"):
        h.decode_attn_partial(qa, cache, torch.tensor([10], dtype=torch.int32, device=DEV))
