"""FP8 weights for the two head projections (DeepSeek-V3 walkthrough, section 4.4: weights in
1 x 128 tiles, high-precision accumulation; section 5.5: FP8 storage with BF16 arithmetic):
mla_absorb_q_fp8 and mla_apply_wuv_fp8 against the oracle on the dequantised weights, every
output, and bit for bit against the bf16 calls given the dequantised weights as bf16 (every
E4M3 value times a power of two is a bf16 number, so the MMAs see the same operands)."""

import numpy as np
import pytest
import torch

import oracle
from mla_latent_kv_28_b200 import binding
from mla_latent_kv_28_b200 import workloads as wl
from tests._parity import assert_close, f64, quantise_weight_e4m3, to_np, workload_np

pytestmark = pytest.mark.gpu

DEV = "cuda:0"


def _deq(codes, exps):
    return oracle.dequantize_weight_fp8(codes.numpy(), exps.numpy().astype(np.int64))


def test_test_quantiser_matches_the_oracle_on_samples():
    w = wl.make_workload(1, 16, [8], seed=70).w_uk
    codes, exps = quantise_weight_e4m3(w)
    rows = to_np(w).reshape(-1, 4, 128)
    rng = np.random.default_rng(1)
    for r, t in zip(rng.integers(0, rows.shape[0], 40), rng.integers(0, 4, 40)):
        assert int(exps[r, t]) == oracle.fp8_row_exponent(rows[r, t])
        ref = oracle.e4m3_encode(oracle.widen(rows[r, t]) / 2.0 ** int(exps[r, t]))
        assert np.array_equal(codes[r, 128 * t:128 * (t + 1)].numpy(), ref)


@pytest.mark.parametrize("batch,n_heads,q_len", [(5, 128, 1), (64, 16, 1), (150, 32, 1), (3, 16, 4)])
def test_fp8_head_projections_every_output(batch, n_heads, q_len):
    w = wl.make_workload(batch, n_heads, [300 + 17 * b for b in range(batch)], seed=71 + batch)
    a = workload_np(w)
    g = w.to(DEV)
    c_uk, e_uk = quantise_weight_e4m3(w.w_uk)
    c_uv, e_uv = quantise_weight_e4m3(w.w_uv)
    w_uk = _deq(c_uk, e_uk)
    w_uv = _deq(c_uv, e_uv)
    h = binding.MlaDecode(n_heads, batch, w.max_kv_len, rope_base=w.rope_base, q_len=q_len)
    if q_len == 1:
        q_c, q_r = g.q_c, g.q_r
    else:
        q_c_h, q_r_h = wl.draw_token_queries(batch, q_len, n_heads, seed=72)
        q_c, q_r = q_c_h.to(DEV), q_r_h.to(DEV)
    q8 = h.absorb_q_fp8(q_c, q_r, c_uk.to(DEV), e_uk.to(DEV), g.kv_lens)
    latent = wl.draw_latent(batch * q_len, n_heads, seed=73).view(tuple(q_c.shape[:-1]) + (512,)).to(DEV)
    o8 = h.apply_wuv_fp8(latent, c_uv.to(DEV), e_uv.to(DEV))
    h.check_device_errors()
    # bit for bit the bf16 calls on the dequantised weights (exact in bf16)
    wb_uk = torch.from_numpy(w_uk).float().to(torch.bfloat16).to(DEV)
    wb_uv = torch.from_numpy(w_uv).float().to(torch.bfloat16).to(DEV)
    assert torch.equal(wb_uk.double().cpu(), torch.from_numpy(w_uk))   # exact
    qb = h.absorb_q(q_c, q_r, wb_uk, g.kv_lens)
    ob = h.apply_wuv(latent, wb_uv)
    h.check_device_errors()
    assert torch.equal(q8.view(torch.int16), qb.view(torch.int16))
    assert torch.equal(o8.view(torch.int16), ob.view(torch.int16))
    # against the oracle on the dequantised weights
    if q_len == 1:
        ref_q = oracle.absorb_query(a["q_c"], a["q_r"], w_uk, a["kv_lens"], w.rope_base)
    else:
        ref_q = oracle.absorb_query_tokens(to_np(q_c_h), to_np(q_r_h), w_uk, a["kv_lens"], w.rope_base)
    assert_close(f64(q8), ref_q, "absorb with FP8 W_UK")
    lat_np = to_np(latent.cpu()).reshape(batch * q_len, n_heads, 512)
    ref_o = oracle.apply_wuv(lat_np, w_uv).reshape(tuple(o8.shape))
    assert_close(f64(o8), ref_o, "W_UV with FP8 weights")
    h.close()


@pytest.mark.parametrize("log2_scale", [-110, 20])
def test_fp8_weight_exponent_ranges(log2_scale):
    """Weights scaled by 2^-110 (tile exponents near the bottom of the range, expanded values
    partly below bf16's normal range) and by 2^20 (exponents above 7: two multiplies per pair
    in the expansion): still bit for bit the bf16 calls on the dequantised weights."""
    batch, n_heads = 9, 32
    w = wl.make_workload(batch, n_heads, [40] * batch, seed=75)
    g = w.to(DEV)
    c_uk, e_uk = quantise_weight_e4m3((w.w_uk.double() * 2.0 ** log2_scale).to(torch.bfloat16))
    c_uv, e_uv = quantise_weight_e4m3((w.w_uv.double() * 2.0 ** log2_scale).to(torch.bfloat16))
    assert (e_uk.min() < -117 and e_uv.min() < -117) if log2_scale < 0 else (e_uk.max() > 7 and e_uv.max() > 7)
    h = binding.MlaDecode(n_heads, batch, w.max_kv_len, rope_base=w.rope_base)
    q8 = h.absorb_q_fp8(g.q_c, g.q_r, c_uk.to(DEV), e_uk.to(DEV), g.kv_lens)
    latent = wl.draw_latent(batch, n_heads, seed=76).to(DEV)
    o8 = h.apply_wuv_fp8(latent, c_uv.to(DEV), e_uv.to(DEV))
    wb_uk = torch.from_numpy(_deq(c_uk, e_uk)).float().to(torch.bfloat16).to(DEV)
    wb_uv = torch.from_numpy(_deq(c_uv, e_uv)).float().to(torch.bfloat16).to(DEV)
    qb = h.absorb_q(g.q_c, g.q_r, wb_uk, g.kv_lens)
    ob = h.apply_wuv(latent, wb_uv)
    h.check_device_errors()
    assert torch.equal(q8.view(torch.int16), qb.view(torch.int16))
    assert torch.equal(o8.view(torch.int16), ob.view(torch.int16))
    h.close()


def test_fp8_weights_whole_step_against_the_nonabsorbed_definition():
    w = wl.make_workload(3, 128, [700, 64, 1500], seed=74)
    a = workload_np(w)
    g = w.to(DEV)
    c_uk, e_uk = quantise_weight_e4m3(w.w_uk)
    c_uv, e_uv = quantise_weight_e4m3(w.w_uv)
    h = binding.MlaDecode(128, 3, w.max_kv_len, rope_base=w.rope_base)
    q_abs = h.absorb_q_fp8(g.q_c, g.q_r, c_uk.to(DEV), e_uk.to(DEV), g.kv_lens)
    latent, _ = h.decode_attn(q_abs, g.cache, g.kv_lens)
    out = h.apply_wuv_fp8(latent, c_uv.to(DEV), e_uv.to(DEV))
    h.check_device_errors()
    ref = oracle.mla_decode_nonabsorbed(a["q_c"], a["q_r"], _deq(c_uk, e_uk), _deq(c_uv, e_uv),
                                        a["cache"], a["kv_lens"], oracle.default_scale(), w.rope_base)
    assert_close(f64(out), ref, "decode step with FP8 W_UK / W_UV")
    h.close()


def test_fp8_weight_arguments_are_checked():
    h = binding.MlaDecode(16, 2, 64)
    q = torch.zeros((2, 16, 128), dtype=torch.bfloat16, device=DEV)
    qr = torch.zeros((2, 16, 64), dtype=torch.bfloat16, device=DEV)
    lens = torch.ones(2, dtype=torch.int32, device=DEV)
    codes = torch.zeros((16 * 128, 512), dtype=torch.uint8, device=DEV)
    exps = torch.zeros((16 * 128, 4), dtype=torch.int8, device=DEV)
    with pytest.raises(ValueError):
        h.absorb_q_fp8(q, qr, codes[:100], exps, lens)
    with pytest.raises(ValueError):
        h.apply_wuv_fp8(torch.zeros((2, 16, 512), dtype=torch.bfloat16, device=DEV), codes, exps[:, :2])
    lib = binding.load_library()
    out = torch.empty((2, 16, 576), dtype=torch.bfloat16, device=DEV)
    st = lib.mla_absorb_q_fp8(h._h, 2, q.data_ptr(), qr.data_ptr(), codes.data_ptr(), None,
                              lens.data_ptr(), out.data_ptr(), None)
    assert st == binding.MLA_ERR_INVALID_ARG
    h.close()
