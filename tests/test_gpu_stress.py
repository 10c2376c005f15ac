"""GPU parity at the edges of the work split and of the numerics: many short sequences (many
segments per cluster, several batch chunks in the head GEMMs), one long sequence cut into as
many splits as there are clusters, a non-default softmax scale, and cache rows whose
magnitudes span four decades (the partial scores cross between the two CTAs of a cluster in
16-bit block floating point). Every check is element by element against the fp64 oracle."""

import numpy as np
import pytest
import torch

import oracle
from mla_latent_kv_28_b200 import binding
from mla_latent_kv_28_b200 import workloads as wl
from tests._parity import assert_close, f64, to_np, workload_np

pytestmark = pytest.mark.gpu

DEV = "cuda:0"


def _handle(w, scale=0.0, max_splits=0):
    return binding.MlaDecode(w.n_heads, w.batch, w.max_kv_len, page_size=w.page_size,
                             softmax_scale=scale, rope_base=w.rope_base, max_splits=max_splits)


def _attention_vs_oracle(w, h, qa, scale, what):
    g = w.to(DEV)
    a = workload_np(w)
    latent, lse = h.decode_attn(qa.to(DEV), g.cache, g.kv_lens, g.page_table)
    h.check_device_errors()
    ref_lat, ref_lse = oracle.latent_attention(to_np(qa), a["cache"], a["kv_lens"], scale,
                                               a["page_table"], a["page_size"])
    assert_close(f64(latent), ref_lat, f"{what}: latent output")
    assert_close(lse.cpu().numpy(), ref_lse, f"{what}: log-sum-exp")


def test_many_short_sequences():
    """300 sequences of 1..200 tokens: a cluster's unit holds several sequences (several
    segments, each with its own query and epilogue), and the head GEMMs run several batch
    chunks (128 sequences per absorb CTA, 64 per W_UV CTA)."""
    w = wl.make_workload(300, 128, ("uniform", 1, 200), seed=21, max_kv_len=200)
    g = w.to(DEV)
    a = workload_np(w)
    h = _handle(w)
    q_abs = h.absorb_q(g.q_c, g.q_r, g.w_uk, g.kv_lens)
    ref_q = oracle.absorb_query(a["q_c"], a["q_r"], a["w_uk"], a["kv_lens"], w.rope_base)
    assert_close(f64(q_abs)[..., :512], ref_q[..., :512], "absorbed query, 300 sequences")
    assert_close(f64(q_abs)[..., 512:], ref_q[..., 512:], "rotated rope query, 300 sequences")
    qa = wl.draw_q_abs(w.batch, w.n_heads, seed=22)
    _attention_vs_oracle(w, h, qa, oracle.default_scale(), "300 short sequences")
    lat_in = wl.draw_latent(w.batch, w.n_heads, seed=23)
    out = h.apply_wuv(lat_in.to(DEV), g.w_uv)
    assert_close(f64(out), oracle.apply_wuv(to_np(lat_in), a["w_uv"]), "W_UV, 300 sequences")


def test_one_long_sequence_in_every_split():
    """One 20,000-token sequence: every cluster takes a few tiles of it, and the combine
    merges as many partials as there are clusters."""
    w = wl.make_workload(1, 128, [20000], seed=24)
    h = _handle(w)
    qa = wl.draw_q_abs(1, 128, seed=25)
    _attention_vs_oracle(w, h, qa, oracle.default_scale(), "20000 tokens, all splits")


def test_nondefault_softmax_scale():
    w = wl.make_workload(2, 64, [300, 77], seed=26)
    h = _handle(w, scale=0.05)
    qa = wl.draw_q_abs(2, 64, seed=27)
    _attention_vs_oracle(w, h, qa, 0.05, "scale 0.05")


def test_cache_rows_spanning_four_decades():
    """Per-token magnitudes 10^U(-2, 2): the largest partial scores of a tile are 10^4 times
    the smallest, the case the 16-bit exchange (scale per head and tile) must carry."""
    w = wl.make_workload(2, 128, [640, 333], seed=28)
    gen = torch.Generator().manual_seed(29)
    mag = torch.pow(10.0, torch.rand((w.cache.shape[0], w.cache.shape[1], 1), generator=gen) * 4 - 2)
    w.cache = (w.cache.float() * mag).to(torch.bfloat16)
    h = _handle(w)
    qa = wl.draw_q_abs(2, 128, seed=30)
    # the scores now reach thousands in the scaled log2 domain: a softmax peaked on a few tokens
    _attention_vs_oracle(w, h, qa, oracle.default_scale(), "four decades of row magnitude")
