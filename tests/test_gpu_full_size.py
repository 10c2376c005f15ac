"""The five named workloads at their full sizes, run the way bench.py runs them (one handle,
automatic split plan), checked on sampled (sequence, head) outputs the oracle computes one
by one, and on properties that hold at any size (every output finite)."""

import numpy as np
import pytest
import torch

import oracle
from mla_latent_kv_28_b200 import binding
from mla_latent_kv_28_b200 import workloads as wl
from tests._parity import assert_close, f64, to_np, workload_np

pytestmark = pytest.mark.gpu

DEV = "cuda:0"

# sampled (sequence, head) pairs per workload: a few sequences, heads spread over 0..n_h-1
SAMPLES = {
    "tiny_h16_l256": None,  # small enough for every output
    "v2_b32_l4096": [(0, 0), (5, 17), (13, 64), (31, 127), (20, 99), (8, 3)],
    "long_b4_l32768": [(0, 1), (1, 50), (2, 100), (3, 127)],
    "single_l131072_lognormal": [(0, 0), (0, 77), (0, 127)],
    "ragged_paged_b64": [(0, 0), (7, 31), (19, 64), (42, 90), (63, 127), (33, 5)],
}


@pytest.mark.parametrize("name", list(SAMPLES))
def test_full_size_workload_sampled_against_oracle(name):
    w = wl.config_workload(name)
    g = w.to(DEV)
    h = binding.MlaDecode(w.n_heads, w.batch, w.max_kv_len, page_size=w.page_size,
                          rope_base=w.rope_base)
    q_abs = h.absorb_q(g.q_c, g.q_r, g.w_uk, g.kv_lens)
    latent, lse = h.decode_attn(q_abs, g.cache, g.kv_lens, g.page_table)
    out = h.apply_wuv(latent, g.w_uv)
    h.check_device_errors()
    assert torch.isfinite(out.float()).all() and torch.isfinite(lse).all()

    a = workload_np(w)
    scale = oracle.default_scale()
    pairs = SAMPLES[name]
    ref = oracle.mla_decode_nonabsorbed(a["q_c"], a["q_r"], a["w_uk"], a["w_uv"], a["cache"],
                                        a["kv_lens"], scale, w.rope_base, a["page_table"],
                                        a["page_size"], pairs=pairs)
    got = f64(out)
    if pairs is None:
        assert_close(got, ref, f"{name}: all outputs")
    else:
        idx = tuple(np.array(pairs).T)
        assert_close(got[idx], ref[idx], f"{name}: sampled outputs")

    # the attention stage alone on one sampled sequence, every head, fed the GPU-independent
    # oracle absorbed query rounded to bf16 (no oracle input comes from the CUDA path)
    b = 0 if pairs is None else pairs[-1][0]
    sel = slice(b, b + 1)
    q_ref = oracle.absorb_query(a["q_c"][sel], a["q_r"][sel], a["w_uk"], a["kv_lens"][sel], w.rope_base)
    q_bf = torch.from_numpy(q_ref).to(torch.bfloat16)
    kv1 = g.kv_lens[sel].contiguous()
    if w.page_size:
        pt1 = g.page_table[sel].contiguous()
        lat1, lse1 = h.decode_attn(q_bf.to(DEV), g.cache, kv1, pt1)
        ref_lat, ref_lse = oracle.latent_attention(to_np(q_bf), a["cache"], a["kv_lens"][sel], scale,
                                                   a["page_table"][sel], w.page_size)
    else:
        lat1, lse1 = h.decode_attn(q_bf.to(DEV), g.cache[sel], kv1)
        ref_lat, ref_lse = oracle.latent_attention(to_np(q_bf), a["cache"][sel], a["kv_lens"][sel], scale)
    h.check_device_errors()
    assert_close(f64(lat1), ref_lat, f"{name}: latent of sequence {b}")
    assert_close(lse1.cpu().numpy(), ref_lse, f"{name}: lse of sequence {b}")
    h.close()
