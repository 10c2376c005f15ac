"""Prefill over the latent cache (mla_prefill_attn): a prompt's T new tokens, 128 attention
rows per work item (one head x 128 consecutive tokens), causal (token t of a sequence with
kv_len rows sees rows 0 .. kv_len - T + t, the MHA equations' softmax over j = 1..t in the
DeepSeek-V2 architecture page). Every output is checked against the fp64 oracle
(latent_attention_tokens) at T = 512 and 2048 with 128 heads, on ragged and paged caches, and
the whole prefill step stage by stage."""

import numpy as np
import pytest
import torch

import oracle
from mla_latent_kv_28_b200 import binding
from mla_latent_kv_28_b200 import workloads as wl
from tests._parity import assert_close, f64, to_np, workload_np

pytestmark = pytest.mark.gpu

DEV = "cuda:0"

CASES = {
    # name: (batch, heads, kv_lens, T, page_size)
    "t512_h128_two_sequences": (2, 128, [512, 700], 512, 0),
    "t2048_h128_prompt_only": (1, 128, [2048], 2048, 0),
    "t300_h16_paged_some_tokens_see_nothing": (3, 16, [300, 1000, 150], 300, 64),
    "t129_h40_long_context": (1, 40, [5000], 129, 0),
}


def _queries(B, T, H, seed):
    return wl.draw_q_abs(B * T, H, seed=seed).view(B, T, H, 576)


def _check_lse(got, ref, what):
    got = np.asarray(got, dtype=np.float64)
    assert np.array_equal(np.isneginf(got), np.isneginf(ref)), f"{what}: tokens without rows"
    fin = np.isfinite(ref)
    assert_close(got[fin], ref[fin], what)


@pytest.mark.parametrize("name", list(CASES))
def test_prefill_every_output_against_oracle(name):
    B, H, lens, T, ps = CASES[name]
    w = wl.make_workload(B, H, lens, page_size=ps, seed=100 + T, max_kv_len=max(lens))
    a = workload_np(w)
    g = w.to(DEV)
    q = _queries(B, T, H, seed=101 + T)
    h = binding.MlaDecode(H, B, w.max_kv_len, page_size=ps, q_len=T)
    lat, lse = h.prefill_attn(q.to(DEV), g.cache, g.kv_lens, g.page_table)
    h.check_device_errors()
    ref_lat, ref_lse = oracle.latent_attention_tokens(to_np(q), a["cache"], a["kv_lens"],
                                                      oracle.default_scale(), a["page_table"], ps)
    assert_close(f64(lat), ref_lat, f"{name}: every latent row")
    _check_lse(lse.cpu().numpy(), ref_lse, f"{name}: every lse")
    h.close()


def test_prefill_matches_the_grouped_decode_call():
    """The same results as mla_decode_attn with the same handle (which runs the T * n_h rows
    in groups of 128 through the split-KV path), within the parity tolerance."""
    w = wl.make_workload(1, 128, [600], seed=110)
    g = w.to(DEV)
    T = 256
    q = _queries(1, T, 128, seed=111).to(DEV)
    h = binding.MlaDecode(128, 1, 600, q_len=T)
    lat_p, lse_p = h.prefill_attn(q, g.cache, g.kv_lens)
    lat_d, lse_d = h.decode_attn(q, g.cache, g.kv_lens)
    h.check_device_errors()
    assert_close(f64(lat_p), f64(lat_d), "prefill vs grouped decode: latent")
    assert_close(lse_p.cpu().numpy(), lse_d.cpu().numpy(), "prefill vs grouped decode: lse")
    h.close()


def test_prefill_step_stage_by_stage():
    """absorb (T tokens) -> prefill attention -> W_UV against the oracle's absorbed stages, each
    fed the oracle's previous stage in bf16; the GPU's own chain against sampled outputs of the
    non-absorbed definition (token t over L rows is a one-token decode over the first
    L - T + t + 1 rows)."""
    B, H, L, T = 1, 128, 700, 384
    w = wl.make_workload(B, H, [L], seed=120)
    a = workload_np(w)
    g = w.to(DEV)
    q_c, q_r = wl.draw_token_queries(B, T, H, seed=121)
    h = binding.MlaDecode(H, B, L, rope_base=w.rope_base, q_len=T)
    q_abs = h.absorb_q(q_c.to(DEV), q_r.to(DEV), g.w_uk, g.kv_lens)
    lat, _ = h.prefill_attn(q_abs, g.cache, g.kv_lens)
    out = h.apply_wuv(lat, g.w_uv)
    h.check_device_errors()
    scale = oracle.default_scale()
    ref_q = oracle.absorb_query_tokens(to_np(q_c), to_np(q_r), a["w_uk"], a["kv_lens"], w.rope_base)
    assert_close(f64(q_abs), ref_q, "absorb of T tokens")
    q_bf = torch.from_numpy(ref_q).float().to(torch.bfloat16)
    lat_s, _ = h.prefill_attn(q_bf.to(DEV), g.cache, g.kv_lens)
    ref_lat, _ = oracle.latent_attention_tokens(to_np(q_bf), a["cache"], a["kv_lens"], scale)
    assert_close(f64(lat_s), ref_lat, "prefill attention")
    lat_bf = torch.from_numpy(ref_lat).float().to(torch.bfloat16)
    out_s = h.apply_wuv(lat_bf.to(DEV), g.w_uv)
    h.check_device_errors()
    ref_o = oracle.apply_wuv(to_np(lat_bf).reshape(B * T, H, 512), a["w_uv"]).reshape(B, T, H, 128)
    assert_close(f64(out_s), ref_o, "W_UV of T tokens")
    got = f64(out)
    for t, i in [(0, 0), (37, 5), (200, 64), (383, 127), (128, 99)]:
        n = L - T + t + 1
        ref = oracle.mla_decode_nonabsorbed(to_np(q_c[:, t]), to_np(q_r[:, t]), a["w_uk"], a["w_uv"],
                                            a["cache"], np.array([n]), scale, w.rope_base,
                                            pairs=[(0, i)])
        assert_close(got[0, t, i], ref[0, i], f"whole prefill step, token {t} head {i}")
    h.close()


def test_prefill_t4096_two_sequences_sampled_tokens():
    """T = 4096 new tokens in each of two sequences (one with 2000 earlier rows), 128 heads:
    sampled tokens, every head, against the oracle's one-token attention over the rows the token
    sees (token t of T over L rows is a one-token decode over the first L - T + t + 1 rows, an
    equivalence the oracle pins fix), plus the first and last token of each 128-token block."""
    T, H = 4096, 128
    w = wl.make_workload(2, H, [4096, 6096], seed=130)
    a = workload_np(w)
    g = w.to(DEV)
    q = _queries(2, T, H, seed=131)
    h = binding.MlaDecode(H, 2, w.max_kv_len, q_len=T)
    lat, lse = h.prefill_attn(q.to(DEV), g.cache, g.kv_lens)
    h.check_device_errors()
    got_lat, got_lse = f64(lat), lse.cpu().numpy()
    qn = to_np(q)
    scale = oracle.default_scale()
    for b, t in [(0, 0), (0, 127), (0, 128), (0, 2047), (0, 4095), (1, 0), (1, 1000), (1, 3968),
                 (1, 4095)]:
        L = int(a["kv_lens"][b])
        n = L - T + t + 1
        rows = a["cache"][b:b + 1]
        ref_lat, ref_lse = oracle.latent_attention(qn[b:b + 1, t], rows, np.array([n]), scale)
        assert_close(got_lat[b, t], ref_lat[0], f"T=4096: sequence {b} token {t}, latent")
        assert_close(got_lse[b, t], ref_lse[0], f"T=4096: sequence {b} token {t}, lse")
    h.close()
