"""The five named workloads at their full sizes, run the way bench.py runs them (one handle,
automatic split plan), with EVERY output checked against the fp64 oracle:

  * a1-a2: every absorbed query row (mla_absorb_q) against oracle.absorb_query;
  * a3-a6: every latent row and log-sum-exp (mla_decode_attn) against oracle.latent_attention,
    both fed the oracle's absorbed query rounded to bf16;
  * a7: every head output (mla_apply_wuv) against oracle.apply_wuv, both fed the oracle's
    latent rounded to bf16;
  * the whole step on the GPU (absorb -> attention -> W_UV, each stage on its own GPU output)
    against the fp64 absorbed path, which the CPU pins hold equal to the non-absorbed
    definition (DeepSeek-V2 paper walkthrough, section 6: absorbed and non-absorbed agree);
  * and the non-absorbed definition itself on sampled (sequence, head) outputs.

No oracle input comes from the CUDA path: each stage is fed the oracle's own previous stage."""

import numpy as np
import pytest
import torch

import oracle
from mla_latent_kv_28_b200 import binding
from mla_latent_kv_28_b200 import workloads as wl
from tests._parity import assert_close, f64, to_np, workload_np

pytestmark = pytest.mark.gpu

DEV = "cuda:0"

# sampled (sequence, head) pairs for the non-absorbed definition (materialising per-head keys
# and values costs d_h times the absorbed path, so it is sampled at full size)
SAMPLES = {
    "tiny_h16_l256": None,  # small enough for every output
    "v2_b32_l4096": [(0, 0), (5, 17), (13, 64), (31, 127), (20, 99), (8, 3)],
    "long_b4_l32768": [(0, 1), (1, 50), (2, 100), (3, 127)],
    "single_l131072_lognormal": [(0, 0), (0, 77), (0, 127)],
    "ragged_paged_b64": [(0, 0), (7, 31), (19, 64), (42, 90), (63, 127), (33, 5)],
}


def _bf16(x: np.ndarray) -> torch.Tensor:
    """fp64 oracle values rounded to bf16 (round to nearest even), on the host."""
    return torch.from_numpy(np.ascontiguousarray(x)).to(torch.float32).to(torch.bfloat16)


@pytest.mark.parametrize("name", list(SAMPLES))
def test_full_size_workload_every_output_against_oracle(name):
    w = wl.config_workload(name)
    g = w.to(DEV)
    a = workload_np(w)
    scale = oracle.default_scale()
    pt, ps = a["page_table"], a["page_size"]
    h = binding.MlaDecode(w.n_heads, w.batch, w.max_kv_len, page_size=w.page_size,
                          rope_base=w.rope_base)

    # the whole step on the GPU, as bench.py runs it
    q_abs = h.absorb_q(g.q_c, g.q_r, g.w_uk, g.kv_lens)
    latent, lse = h.decode_attn(q_abs, g.cache, g.kv_lens, g.page_table)
    out = h.apply_wuv(latent, g.w_uv)
    h.check_device_errors()

    # a1-a2: every absorbed query row
    q_ref = oracle.absorb_query(a["q_c"], a["q_r"], a["w_uk"], a["kv_lens"], w.rope_base)
    assert_close(f64(q_abs), q_ref, f"{name}: every absorbed query row")

    # a3-a6: every latent row and lse, from the oracle's absorbed query in bf16
    q_bf = _bf16(q_ref)
    lat_s, lse_s = h.decode_attn(q_bf.to(DEV), g.cache, g.kv_lens, g.page_table)
    h.check_device_errors()
    ref_lat, ref_lse = oracle.latent_attention(to_np(q_bf), a["cache"], a["kv_lens"], scale, pt, ps)
    assert_close(f64(lat_s), ref_lat, f"{name}: every latent row")
    assert_close(lse_s.cpu().numpy(), ref_lse, f"{name}: every lse")

    # a7: every head output, from the oracle's latent in bf16
    lat_bf = _bf16(ref_lat)
    out_s = h.apply_wuv(lat_bf.to(DEV), g.w_uv)
    h.check_device_errors()
    assert_close(f64(out_s), oracle.apply_wuv(to_np(lat_bf), a["w_uv"]), f"{name}: every W_UV output")

    # the whole GPU step against the fp64 absorbed path (no rounding between its stages)
    ref_out, ref_lat64, ref_lse64 = oracle.mla_decode_absorbed(
        a["q_c"], a["q_r"], a["w_uk"], a["w_uv"], a["cache"], a["kv_lens"], scale, w.rope_base,
        pt, ps)
    assert torch.isfinite(out.float()).all() and torch.isfinite(lse).all()
    assert_close(f64(out), ref_out, f"{name}: every output of the whole step")
    assert_close(f64(latent), ref_lat64, f"{name}: every latent row of the whole step")
    assert_close(lse.cpu().numpy(), ref_lse64, f"{name}: every lse of the whole step")

    # the non-absorbed definition (per-head keys and values materialised)
    pairs = SAMPLES[name]
    ref_na = oracle.mla_decode_nonabsorbed(a["q_c"], a["q_r"], a["w_uk"], a["w_uv"], a["cache"],
                                           a["kv_lens"], scale, w.rope_base, pt, ps, pairs=pairs)
    got = f64(out)
    if pairs is None:
        assert_close(got, ref_na, f"{name}: all outputs vs the non-absorbed definition")
    else:
        idx = tuple(np.array(pairs).T)
        assert_close(got[idx], ref_na[idx], f"{name}: sampled outputs vs the non-absorbed definition")
    h.close()
