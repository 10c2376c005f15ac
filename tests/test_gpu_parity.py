"""GPU parity: every entry point of the C ABI against the fp64 oracle, element by element,
at sizes that span several 64-token tiles and ragged tails; plus the invariances and
device-side checks of the decode path. Needs a B200 and the built library."""

import math

import numpy as np
import pytest
import torch

import oracle
from mla_latent_kv_28_b200 import binding
from mla_latent_kv_28_b200 import workloads as wl
from tests._parity import assert_close, f64, to_np, workload_np

pytestmark = pytest.mark.gpu

DEV = "cuda:0"


def _handle(w, max_splits=0, scale=0.0):
    return binding.MlaDecode(w.n_heads, w.batch, w.max_kv_len, page_size=w.page_size,
                             softmax_scale=scale, rope_base=w.rope_base, max_splits=max_splits)


def _run_step(w, max_splits=0):
    g = w.to(DEV)
    h = _handle(w, max_splits)
    q_abs = h.absorb_q(g.q_c, g.q_r, g.w_uk, g.kv_lens)
    latent, lse = h.decode_attn(q_abs, g.cache, g.kv_lens, g.page_table)
    out = h.apply_wuv(latent, g.w_uv)
    h.check_device_errors()
    return q_abs, latent, lse, out


def _oracle_full(w):
    a = workload_np(w)
    scale = oracle.default_scale()
    ref = oracle.mla_decode_nonabsorbed(a["q_c"], a["q_r"], a["w_uk"], a["w_uv"], a["cache"],
                                        a["kv_lens"], scale, w.rope_base, a["page_table"],
                                        a["page_size"])
    return ref


SMALL_CASES = {
    "one_seq_h16_ragged": dict(batch=1, n_heads=16, kv_lens=[200], rope_base=0.0),
    "h16_rope_lens": dict(batch=3, n_heads=16, kv_lens=[1, 64, 333], rope_base=10000.0),
    "h128_ragged": dict(batch=3, n_heads=128, kv_lens=[65, 130, 191], rope_base=10000.0),
    "h40_odd_heads": dict(batch=2, n_heads=40, kv_lens=[129, 7], rope_base=10000.0),
    "paged_h128": dict(batch=4, n_heads=128, kv_lens=[1, 64, 200, 333], page_size=64,
                       rope_base=10000.0, max_kv_len=512),
    "with_empty_sequence": dict(batch=3, n_heads=32, kv_lens=[100, 0, 70], rope_base=10000.0),
}


@pytest.mark.parametrize("case", sorted(SMALL_CASES))
def test_whole_step_matches_nonabsorbed_oracle(case):
    w = wl.make_workload(seed=7, name=case, **SMALL_CASES[case])
    _, _, _, out = _run_step(w)
    assert_close(f64(out), _oracle_full(w), f"{case}: head outputs")


@pytest.mark.parametrize("case", ["h16_rope_lens", "h128_ragged", "paged_h128"])
def test_each_entry_point_matches_its_oracle_stage(case):
    w = wl.make_workload(seed=8, name=case, **SMALL_CASES[case])
    g = w.to(DEV)
    a = workload_np(w)
    h = _handle(w)
    # absorb: GPU q_abs vs the oracle's fp64 absorbed query
    q_abs = h.absorb_q(g.q_c, g.q_r, g.w_uk, g.kv_lens)
    ref_q = oracle.absorb_query(a["q_c"], a["q_r"], a["w_uk"], a["kv_lens"], w.rope_base)
    assert_close(f64(q_abs)[..., :512], ref_q[..., :512], "absorbed query")
    assert_close(f64(q_abs)[..., 512:], ref_q[..., 512:], "rotated rope query")
    # attention alone, on a drawn bf16 absorbed query
    qa = wl.draw_q_abs(w.batch, w.n_heads, seed=3)
    latent, lse = h.decode_attn(qa.to(DEV), g.cache, g.kv_lens, g.page_table)
    ref_lat, ref_lse = oracle.latent_attention(to_np(qa), a["cache"], a["kv_lens"],
                                               oracle.default_scale(), a["page_table"],
                                               a["page_size"])
    assert_close(f64(latent), ref_lat, "latent output")
    assert_close(lse.cpu().numpy(), ref_lse, "log-sum-exp")
    # W_UV alone, on a drawn bf16 latent
    lat_in = wl.draw_latent(w.batch, w.n_heads, seed=4)
    out = h.apply_wuv(lat_in.to(DEV), g.w_uv)
    assert_close(f64(out), oracle.apply_wuv(to_np(lat_in), a["w_uv"]), "W_UV output")
    h.check_device_errors()


def test_rope_position_follows_kv_len():
    """The query is rotated at position kv_len-1: compare a long and a short sequence."""
    w = wl.make_workload(2, 8, [4097, 3], rope_base=10000.0, seed=9)
    g = w.to(DEV)
    h = _handle(w)
    q_abs = h.absorb_q(g.q_c, g.q_r, g.w_uk, g.kv_lens)
    ref = oracle.absorb_query(to_np(w.q_c), to_np(w.q_r), to_np(w.w_uk), w.kv_lens.numpy(), 10000.0)
    assert_close(f64(q_abs)[..., 512:], ref[..., 512:], "rope at 4096 and 2")


def test_split_count_does_not_change_the_result():
    w = wl.make_workload(2, 128, [1000, 3000], seed=10)
    outs = []
    for ms in (1, 2, 7, 0):
        _, latent, lse, out = _run_step(w, max_splits=ms)
        outs.append((f64(latent), lse.cpu().numpy()))
    for lat, lse in outs[1:]:
        assert np.max(np.abs(lat - outs[0][0])) <= 2e-2 * np.max(np.abs(outs[0][0]))
        np.testing.assert_allclose(lse, outs[0][1], atol=1e-4, rtol=1e-5)


def test_paged_equals_contiguous_bit_for_bit_and_page_order_is_irrelevant():
    lens = [70, 300, 1]
    wp = wl.make_workload(3, 64, lens, page_size=64, seed=11, max_kv_len=320)
    # the same logical rows, laid out contiguously
    cont = torch.full((3, 320, 576), float("nan"), dtype=torch.bfloat16)
    for b, L in enumerate(lens):
        for j in range(L):
            cont[b, j] = wp.cache[int(wp.page_table[b, j // 64]), j % 64]
    wc = wl.Workload("cont", 3, 64, wp.kv_lens, wp.q_c, wp.q_r, wp.w_uk, wp.w_uv, cont, None, 0,
                     wp.rope_base, 320)
    _, lat_p, lse_p, out_p = _run_step(wp, max_splits=1)
    _, lat_c, lse_c, out_c = _run_step(wc, max_splits=1)
    assert torch.equal(out_p.view(torch.int16), out_c.view(torch.int16))
    assert torch.equal(lse_p, lse_c)
    # permute the physical pages and rewrite the table: identical output
    perm = torch.randperm(wp.num_pages, generator=torch.Generator().manual_seed(5))
    inv = torch.empty_like(perm)
    inv[perm] = torch.arange(wp.num_pages)
    cache2 = wp.cache[perm]
    table2 = torch.where(wp.page_table >= 0, inv[wp.page_table.clamp(min=0).long()].to(torch.int32),
                         wp.page_table)
    wp2 = wl.Workload("perm", 3, 64, wp.kv_lens, wp.q_c, wp.q_r, wp.w_uk, wp.w_uv, cache2, table2,
                      64, wp.rope_base, 320)
    _, _, _, out_p2 = _run_step(wp2, max_splits=1)
    assert torch.equal(out_p.view(torch.int16), out_p2.view(torch.int16))


def test_deterministic():
    w = wl.make_workload(2, 128, [777, 1500], seed=12)
    a = _run_step(w)[3]
    b = _run_step(w)[3]
    assert torch.equal(a.view(torch.int16), b.view(torch.int16))


def test_nan_rows_outside_sequences_never_reach_the_output():
    w = wl.make_workload(4, 128, [1, 63, 65, 500], page_size=64, seed=13, max_kv_len=512,
                         spare_pages=7)
    _, latent, lse, out = _run_step(w)
    assert torch.isfinite(out.float()).all() and torch.isfinite(latent.float()).all()
    assert torch.isfinite(lse).all()


def test_empty_sequence_gives_zero_and_minus_inf():
    w = wl.make_workload(2, 16, [0, 5], seed=14)
    _, latent, lse, out = _run_step(w)
    assert torch.count_nonzero(latent[0]) == 0 and torch.count_nonzero(out[0]) == 0
    assert torch.isneginf(lse[0]).all() and torch.isfinite(lse[1]).all()


def test_bad_page_entry_sets_the_error_word_and_is_skipped():
    w = wl.make_workload(2, 16, [100, 100], page_size=64, seed=15, max_kv_len=128)
    g = w.to(DEV)
    bad = g.page_table.clone()
    bad[1, 1] = w.num_pages + 3
    h = _handle(w)
    q_abs = h.absorb_q(g.q_c, g.q_r, g.w_uk, g.kv_lens)
    latent, _ = h.decode_attn(q_abs, g.cache, g.kv_lens, bad)
    with pytest.raises(binding.MlaError) as e:
        h.check_device_errors()
    assert e.value.status == binding.MLA_ERR_DEVICE_CHECK and e.value.detail & binding.ERR_BAD_PAGE
    assert torch.isfinite(latent.float()).all()
    h.check_device_errors()  # cleared by the read


def test_kv_len_beyond_the_maximum_sets_the_error_word():
    w = wl.make_workload(1, 16, [64], seed=16)
    g = w.to(DEV)
    h = binding.MlaDecode(16, 1, 64, rope_base=w.rope_base)
    q_abs = h.absorb_q(g.q_c, g.q_r, g.w_uk, g.kv_lens)
    too_long = torch.tensor([65], dtype=torch.int32, device=DEV)
    h.decode_attn(q_abs, g.cache, too_long)
    with pytest.raises(binding.MlaError) as e:
        h.check_device_errors()
    assert e.value.detail & binding.ERR_BAD_KV_LEN


def test_invalid_arguments_are_rejected_on_the_host():
    w = wl.make_workload(2, 16, [10, 20], seed=17).to(DEV)
    h = _handle(w)
    q_abs = h.absorb_q(w.q_c, w.q_r, w.w_uk, w.kv_lens)
    lib = binding.load_library()
    out = torch.empty((2, 16, 512), dtype=torch.bfloat16, device=DEV)
    s = torch.cuda.current_stream().cuda_stream
    c = w.cache.data_ptr()
    # batch beyond max_batch, odd row stride, seq_stride below max_kv_len, misaligned pointer
    for args in [(3, 576, 20, c), (2, 577, 20, c), (2, 576, 5, c), (2, 576, 20, c + 2)]:
        st = lib.mla_decode_attn(h._h, args[0], q_abs.data_ptr(), args[3], c + 1024, args[1], args[2],
                                 w.kv_lens.data_ptr(), None, 0, 0, out.data_ptr(), None, s)
        assert st == binding.MLA_ERR_INVALID_ARG
    # a page table given to a contiguous handle
    st = lib.mla_decode_attn(h._h, 2, q_abs.data_ptr(), c, c + 1024, 576, 20, w.kv_lens.data_ptr(),
                             w.kv_lens.data_ptr(), 1, 1, out.data_ptr(), None, s)
    assert st == binding.MLA_ERR_INVALID_ARG
    h.check_device_errors()


def test_one_token_sequence_returns_its_latent_row():
    w = wl.make_workload(2, 128, [1, 1], seed=18)
    g = w.to(DEV)
    h = _handle(w)
    latent, lse = h.decode_attn(wl.draw_q_abs(2, 128).to(DEV), g.cache, g.kv_lens)
    ref = w.cache[:, 0, :512].float()
    assert torch.equal(latent.cpu().float(), ref[:, None, :].expand(2, 128, 512))
