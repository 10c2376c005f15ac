"""GPU parity with YaRN on (DeepSeek-V2's s = 40, alpha = 1, beta = 32, 4K original context,
sqrt(t) = 0.0707 ln s + 1): the rotated query at positions up to 128K, the written key, and a
whole decode step with the default (YaRN-scaled) softmax scale, each against the fp64 oracle
given the same YaRN parameters."""

import numpy as np
import pytest
import torch

import oracle
from mla_latent_kv_28_b200 import binding
from mla_latent_kv_28_b200 import workloads as wl
from tests._parity import assert_close, f64, to_np, workload_np

pytestmark = pytest.mark.gpu

DEV = "cuda:0"
YARN = dict(yarn_factor=40.0, yarn_original_len=4096, yarn_alpha=1.0, yarn_beta=32.0,
            yarn_mscale_coef=0.0707)
Y = oracle.Yarn(factor=40.0, original_len=4096, alpha=1.0, beta=32.0, mscale_coef=0.0707)


def test_absorbed_query_rotated_with_yarn_at_long_positions():
    # the absorption reads only the lengths, so a small cache stands beside long lengths
    w = wl.make_workload(4, 16, [1, 2, 3, 4], seed=61)
    w.kv_lens = torch.tensor([1, 4097, 65536, 131072], dtype=torch.int32)
    h = binding.MlaDecode(16, 4, 131072, **YARN)
    g_qc, g_qr, g_wuk = w.q_c.to(DEV), w.q_r.to(DEV), w.w_uk.to(DEV)
    lens = w.kv_lens.to(DEV)
    q_abs = h.absorb_q(g_qc, g_qr, g_wuk, lens)
    h.check_device_errors()
    ref = oracle.absorb_query(to_np(w.q_c), to_np(w.q_r), to_np(w.w_uk), w.kv_lens.numpy(),
                              w.rope_base, Y)
    assert_close(f64(q_abs)[..., 512:], ref[..., 512:], "YaRN-rotated q^R")
    assert_close(f64(q_abs)[..., :512], ref[..., :512], "absorbed q (unchanged by YaRN)")
    plain = oracle.absorb_query(to_np(w.q_c), to_np(w.q_r), to_np(w.w_uk), w.kv_lens.numpy(),
                                w.rope_base)
    # the check can tell YaRN from plain RoPE at these positions
    assert np.max(np.abs(plain[1:, :, 512:] - ref[1:, :, 512:])) > 0.5


def test_written_key_rotated_with_yarn():
    """The cache write at positions 99,999 and 7: a paged cache whose table points only the
    pages of the new tokens at real pages."""
    B, P = 2, 4
    cache = torch.full((P, 64, 576), float("nan"), dtype=torch.bfloat16, device=DEV)
    lens = torch.tensor([100000, 8], dtype=torch.int32, device=DEV)
    table = torch.full((B, 131072 // 64), -1, dtype=torch.int32, device=DEV)
    table[0, 99999 // 64] = 2
    table[1, 0] = 1
    inp = wl.draw_append_inputs(B, 1024, seed=62)
    h = binding.MlaDecode(16, B, 131072, page_size=64, **YARN)
    dev = {k: v.to(DEV) for k, v in inp.items()}
    h.append_kv(dev["hidden"], dev["w_dkv"], dev["w_kr"], dev["gamma"], cache, lens, table)
    h.check_device_errors()
    ref = oracle.cache_rows(to_np(inp["hidden"]), to_np(inp["w_dkv"]), to_np(inp["w_kr"]),
                            to_np(inp["gamma"]), [100000, 8], 10000.0, 1e-6, Y)
    got = np.stack([f64(cache[2, 99999 % 64]), f64(cache[1, 7])])
    assert_close(got[:, 512:], ref[:, 512:], "YaRN-rotated k^R")
    assert_close(got[:, :512], ref[:, :512], "c^KV (unchanged by YaRN)")


def test_decode_step_with_yarn_and_its_default_scale():
    w = wl.make_workload(3, 32, [3000, 777, 64], seed=63)
    g = w.to(DEV)
    a = workload_np(w)
    h = binding.MlaDecode(32, 3, w.max_kv_len, **YARN)
    q_abs = h.absorb_q(g.q_c, g.q_r, g.w_uk, g.kv_lens)
    latent, lse = h.decode_attn(q_abs, g.cache, g.kv_lens)
    out = h.apply_wuv(latent, g.w_uv)
    h.check_device_errors()
    scale = oracle.default_scale(yarn=Y)
    ref_out = oracle.mla_decode_nonabsorbed(a["q_c"], a["q_r"], a["w_uk"], a["w_uv"], a["cache"],
                                            a["kv_lens"], scale, w.rope_base, yarn=Y)
    assert_close(f64(out), ref_out, "YaRN decode step: head outputs")
    ref_q = oracle.absorb_query(a["q_c"], a["q_r"], a["w_uk"], a["kv_lens"], w.rope_base, Y)
    _, ref_lse = oracle.latent_attention(ref_q, a["cache"], a["kv_lens"], scale)
    assert_close(lse.cpu().numpy(), ref_lse, "YaRN decode step: log-sum-exp (scale t/sqrt(192))")
