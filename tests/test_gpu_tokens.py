"""GPU parity with several new tokens per sequence (multi-token prediction / speculative
decoding): the T new tokens are the last T cached rows, token t attends to the rows up to its
own position and its q^R is rotated there. Every check is against the fp64 oracle."""

import numpy as np
import pytest
import torch

import oracle
from mla_latent_kv_28_b200 import binding
from mla_latent_kv_28_b200 import workloads as wl
from tests._parity import assert_close, f64, to_np, workload_np

pytestmark = pytest.mark.gpu

DEV = "cuda:0"


def _step_vs_oracle(n_h, T, lens, page_size, seed, max_kv_len=None):
    w = wl.make_workload(len(lens), n_h, lens, page_size=page_size, seed=seed, max_kv_len=max_kv_len)
    q_c, q_r = wl.draw_token_queries(len(lens), T, n_h, seed=seed + 1)
    g = w.to(DEV)
    a = workload_np(w)
    h = binding.MlaDecode(n_h, len(lens), w.max_kv_len, page_size=page_size, q_len=T)
    q_abs = h.absorb_q(q_c.to(DEV), q_r.to(DEV), g.w_uk, g.kv_lens)
    latent, lse = h.decode_attn(q_abs, g.cache, g.kv_lens, g.page_table)
    out = h.apply_wuv(latent, g.w_uv)
    h.check_device_errors()
    assert tuple(out.shape) == (len(lens), T, n_h, 128)
    ref_q = oracle.absorb_query_tokens(to_np(q_c), to_np(q_r), a["w_uk"], a["kv_lens"], w.rope_base)
    assert_close(f64(q_abs)[..., 512:], ref_q[..., 512:], f"T={T}: rotated q^R per token")
    ref_lat, ref_lse = oracle.latent_attention_tokens(to_np(q_abs), a["cache"], a["kv_lens"],
                                                      oracle.default_scale(), a["page_table"],
                                                      a["page_size"])
    got_lse = lse.cpu().numpy()
    assert np.array_equal(np.isneginf(got_lse), np.isneginf(ref_lse)), "tokens without rows"
    fin = np.isfinite(ref_lse)
    assert_close(got_lse[fin], ref_lse[fin], f"T={T}: log-sum-exp")
    assert_close(f64(latent), ref_lat, f"T={T}: latent output")
    ref_out = oracle.mla_decode_nonabsorbed_tokens(to_np(q_c), to_np(q_r), a["w_uk"], a["w_uv"],
                                                   a["cache"], a["kv_lens"], oracle.default_scale(),
                                                   w.rope_base, a["page_table"], a["page_size"])
    assert_close(f64(out), ref_out, f"T={T}: head outputs")


def test_eight_tokens_sixteen_heads_contiguous():
    """128 attention rows (8 tokens x 16 heads); a sequence shorter than T (its first tokens
    see nothing), one inside a tile, one over several tiles."""
    _step_vs_oracle(16, 8, [8, 100, 700, 3], 0, 70)


def test_two_tokens_all_128_heads_in_two_row_groups():
    """DeepSeek-V2's 128 heads with 2 new tokens: 256 attention rows, run as two groups of 128
    over the same cache and plan."""
    _step_vs_oracle(128, 2, [300, 64, 1000], 0, 76)


def test_five_tokens_64_heads_uneven_groups():
    """320 rows: groups of 128, 128 and 64, on a paged cache."""
    _step_vs_oracle(64, 5, [5, 129, 700], 64, 77, max_kv_len=700)


def test_two_tokens_paged_ragged():
    _step_vs_oracle(32, 2, [int(x) for x in np.random.default_rng(71).integers(1, 500, 20)], 64, 72,
                    max_kv_len=500)


def test_two_tokens_one_long_sequence_in_every_split():
    """64 heads x 2 tokens over 20,000 rows: the per-row limit holds in every split and the
    combine merges them."""
    w = wl.make_workload(1, 64, [20000], seed=73)
    g = w.to(DEV)
    a = workload_np(w)
    qa = wl.draw_q_abs(1, 128, seed=74).view(1, 2, 64, 576)
    h = binding.MlaDecode(64, 1, 20000, q_len=2)
    latent, lse = h.decode_attn(qa.to(DEV), g.cache, g.kv_lens)
    h.check_device_errors()
    ref_lat, ref_lse = oracle.latent_attention_tokens(to_np(qa), a["cache"], a["kv_lens"],
                                                      oracle.default_scale())
    assert_close(f64(latent), ref_lat, "T=2, 20000 rows: latent")
    assert_close(lse.cpu().numpy(), ref_lse, "T=2, 20000 rows: lse")


def test_cache_write_of_three_new_tokens():
    """hidden [B, 3, d]: the rows at L-3, L-2, L-1, each rotated at its own position."""
    lens = [3, 64, 130]
    w = wl.make_workload(3, 16, lens, seed=75)
    g = w.to(DEV)
    before = g.cache.clone()
    inp = wl.draw_append_inputs(9, 1024, seed=76)
    hidden = inp["hidden"].view(3, 3, 1024)
    h = binding.MlaDecode(16, 3, w.max_kv_len, q_len=3)
    h.append_kv(hidden.to(DEV), inp["w_dkv"].to(DEV), inp["w_kr"].to(DEV), inp["gamma"].to(DEV),
                g.cache, g.kv_lens)
    h.check_device_errors()
    # the oracle's cache row of a token at position p is cache_rows with kv_len p + 1
    row_lens = [L - 3 + t + 1 for L in lens for t in range(3)]
    ref = oracle.cache_rows(to_np(inp["hidden"]), to_np(inp["w_dkv"]), to_np(inp["w_kr"]),
                            to_np(inp["gamma"]), row_lens, w.rope_base)
    got = np.stack([f64(g.cache[b, lens[b] - 3 + t]) for b in range(3) for t in range(3)])
    assert_close(got, ref, "three new tokens' cache rows")
    mask = torch.ones(g.cache.shape[:2], dtype=torch.bool, device=DEV)
    for b in range(3):
        mask[b, lens[b] - 3:lens[b]] = False
    assert torch.equal(g.cache.view(torch.int16)[mask], before.view(torch.int16)[mask])
