"""mla_decode_step, the whole decode step in one call (the absorption kernel builds the
split-KV work plan in one extra block instead of the plan's own launch): bit for bit the
three calls mla_absorb_q -> mla_decode_attn -> mla_apply_wuv on the same inputs (the same
kernels on the same plan), for contiguous and paged caches, an empty sequence, capped and
balanced plans, more sequences than one absorption tile holds, several new tokens per
sequence, and against the fp64 oracle; arguments are checked before anything is launched."""

import pytest
import torch

from mla_latent_kv_28_b200 import binding
from mla_latent_kv_28_b200 import workloads as wl
from tests._parity import assert_close, f64, workload_np

import oracle

pytestmark = pytest.mark.gpu

DEV = "cuda:0"

CASES = {
    "contiguous_h128": (dict(batch=3, n_heads=128, kv_lens=[700, 333, 64]), 0),
    "paged_ragged_with_empty": (dict(batch=20, n_heads=64, kv_lens=[0] + [37 * i + 1 for i in range(19)],
                                     page_size=64, max_kv_len=704), 0),
    "capped_plan": (dict(batch=5, n_heads=32, kv_lens=[1, 500, 129, 64, 1000]), 3),
    "150_sequences": (dict(batch=150, n_heads=16, kv_lens=("uniform", 1, 300), max_kv_len=300), 0),
}


def _three_calls(h, g, q_c, q_r):
    q_abs = h.absorb_q(q_c, q_r, g.w_uk, g.kv_lens)
    latent, _ = h.decode_attn(q_abs, g.cache, g.kv_lens, g.page_table, want_lse=False)
    return q_abs, latent, h.apply_wuv(latent, g.w_uv)


@pytest.mark.parametrize("case", sorted(CASES))
def test_step_equals_the_three_calls(case):
    spec, max_splits = CASES[case]
    w = wl.make_workload(seed=41, name=case, **spec)
    g = w.to(DEV)
    h = binding.MlaDecode(w.n_heads, w.batch, w.max_kv_len, page_size=w.page_size,
                          rope_base=w.rope_base, max_splits=max_splits)
    q_abs, latent, out = _three_calls(h, g, g.q_c, g.q_r)
    bufs = dict(q_abs=torch.full_like(q_abs, float("nan")), latent=torch.full_like(latent, float("nan")),
                out=torch.full_like(out, float("nan")))
    out_s = h.step(g.q_c, g.q_r, g.w_uk, g.w_uv, g.cache, g.kv_lens, g.page_table, bufs=bufs)
    h.check_device_errors()
    assert torch.equal(bufs["q_abs"].view(torch.int16), q_abs.view(torch.int16)), f"{case}: q_abs"
    assert torch.equal(bufs["latent"].view(torch.int16), latent.view(torch.int16)), f"{case}: latent"
    assert torch.equal(out_s.view(torch.int16), out.view(torch.int16)), f"{case}: head outputs"
    if case == "contiguous_h128":
        a = workload_np(w)
        ref = oracle.mla_decode_nonabsorbed(a["q_c"], a["q_r"], a["w_uk"], a["w_uv"], a["cache"],
                                            a["kv_lens"], oracle.default_scale(), w.rope_base)
        assert_close(f64(out_s), ref, f"{case}: step vs the non-absorbed definition")
    h.close()


def test_step_with_two_new_tokens_per_sequence():
    w = wl.make_workload(4, 32, [90, 300, 2, 65], seed=43)
    g = w.to(DEV)
    h = binding.MlaDecode(32, 4, w.max_kv_len, rope_base=w.rope_base, q_len=2)
    q_c, q_r = (t.to(DEV) for t in wl.draw_token_queries(4, 2, 32, seed=44))
    _, _, out = _three_calls(h, g, q_c, q_r)
    out_s = h.step(q_c, q_r, g.w_uk, g.w_uv, g.cache, g.kv_lens)
    h.check_device_errors()
    assert out_s.shape == (4, 2, 32, 128)
    assert torch.equal(out_s.view(torch.int16), out.view(torch.int16))
    h.close()


def test_step_arguments_are_checked_before_any_launch():
    w = wl.make_workload(2, 16, [10, 20], seed=45)
    g = w.to(DEV)
    h = binding.MlaDecode(16, 2, w.max_kv_len)
    lib = binding.load_library()
    q_abs = torch.empty((2, 16, 576), dtype=torch.bfloat16, device=DEV)
    latent = torch.empty((2, 16, 512), dtype=torch.bfloat16, device=DEV)
    out = torch.full((2, 16, 128), 7.0, dtype=torch.bfloat16, device=DEV)
    row_stride, seq_stride = g.cache.stride(1), g.cache.stride(0) // g.cache.stride(1)
    c_kv, k_r = g.cache.data_ptr(), g.cache.data_ptr() + 1024

    def call(**over):
        a = dict(q_c=g.q_c.data_ptr(), q_abs=q_abs.data_ptr(), latent=latent.data_ptr(),
                 seq_stride=seq_stride, batch=2)
        a.update(over)
        return lib.mla_decode_step(h._h, a["batch"], a["q_c"], g.q_r.data_ptr(), g.w_uk.data_ptr(),
                                   g.w_uv.data_ptr(), c_kv, k_r, row_stride, a["seq_stride"],
                                   g.kv_lens.data_ptr(), None, 0, 0, a["q_abs"], a["latent"],
                                   out.data_ptr(), None)

    assert call(q_c=None) == binding.MLA_ERR_INVALID_ARG
    assert call(latent=None) == binding.MLA_ERR_INVALID_ARG
    assert call(q_abs=q_abs.data_ptr() + 2) == binding.MLA_ERR_INVALID_ARG   # not 16-byte aligned
    assert call(seq_stride=1) == binding.MLA_ERR_INVALID_ARG                 # below max_kv_len
    assert call(batch=3) == binding.MLA_ERR_INVALID_ARG                      # above max_batch
    torch.cuda.synchronize()
    assert bool((out == 7.0).all()), "a rejected call wrote its output"
    assert call() == binding.MLA_OK
    h.check_device_errors()
    assert not bool((out == 7.0).all())
    h.close()
