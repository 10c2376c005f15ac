"""GPU parity of the attention over a quantised cache (E4M3 codes, one power-of-two scale per
row): against the fp64 oracle over the dequantised rows, and bit for bit against the bf16
attention over those same rows (the expansion to bf16 is exact, so the two must agree)."""

import numpy as np
import pytest
import torch

import oracle
from mla_latent_kv_28_b200 import binding
from mla_latent_kv_28_b200 import workloads as wl
from tests._parity import assert_close, f64, to_np, workload_np

pytestmark = pytest.mark.gpu

DEV = "cuda:0"


def _quantise(cache: torch.Tensor):
    """bf16 cache [N1, N2, 576] -> (codes uint8, exps int8, dequantised bf16 cache). Rows that
    are not part of a sequence (NaN in the workload) become NaN codes with exponent 0, so any
    read of them would show. Exponents from the oracle; codes by torch's E4M3 cast, which the
    oracle pins rounding for rounding."""
    rows = oracle.widen(to_np(cache)).reshape(-1, 576)
    valid = np.isfinite(rows).all(axis=1)
    exps = np.zeros(rows.shape[0], dtype=np.int8)
    codes = np.full(rows.shape, 0x7F, dtype=np.uint8)
    idx = np.nonzero(valid)[0]
    e = np.array([oracle.fp8_row_exponent(rows[i]) for i in idx], dtype=np.int64)
    exps[idx] = e
    scaled = torch.from_numpy(rows[idx] / np.exp2(e)[:, None]).to(torch.float32)
    codes[idx] = scaled.to(torch.float8_e4m3fn).view(torch.uint8).numpy()
    deq = np.full(rows.shape, np.nan)
    deq[idx] = oracle.dequantize_rows_fp8(codes[idx], exps[idx])
    shape = cache.shape
    return (torch.from_numpy(codes).view(shape), torch.from_numpy(exps).view(shape[:2]),
            torch.from_numpy(deq).to(torch.bfloat16).view(shape), deq.reshape(shape))


def _check(w, qa, what, max_splits=0):
    g = w.to(DEV)
    a = workload_np(w)
    codes, exps, deq_bf16, deq64 = _quantise(w.cache)
    h = binding.MlaDecode(w.n_heads, w.batch, w.max_kv_len, page_size=w.page_size,
                          max_splits=max_splits)
    lat8, lse8 = h.decode_attn_fp8(qa.to(DEV), codes.to(DEV), exps.to(DEV), g.kv_lens, g.page_table)
    h.check_device_errors()
    ref_lat, ref_lse = oracle.latent_attention(to_np(qa), deq64, a["kv_lens"], oracle.default_scale(),
                                               a["page_table"], a["page_size"])
    assert_close(f64(lat8), ref_lat, f"{what}: latent")
    assert_close(lse8.cpu().numpy(), ref_lse, f"{what}: lse")
    lat16, lse16 = h.decode_attn(qa.to(DEV), deq_bf16.to(DEV), g.kv_lens, g.page_table)
    h.check_device_errors()
    assert torch.equal(lat8, lat16), f"{what}: quantised and bf16 paths differ"
    assert torch.equal(lse8, lse16), f"{what}: quantised and bf16 log-sum-exp differ"


def test_contiguous_three_sequences():
    w = wl.make_workload(3, 128, [700, 333, 64], seed=90)
    _check(w, wl.draw_q_abs(3, 128, seed=91), "contiguous")


def test_paged_ragged():
    lens = [int(x) for x in np.random.default_rng(92).integers(1, 500, 20)]
    w = wl.make_workload(20, 64, lens, page_size=64, seed=93, max_kv_len=500)
    _check(w, wl.draw_q_abs(20, 64, seed=94), "paged ragged")


def test_many_short_sequences_many_segments():
    """300 sequences of 1..200 tokens: several segments per cluster, each expanded tile
    interleaved with the query loads and epilogues of the transition warpgroup."""
    w = wl.make_workload(300, 32, ("uniform", 1, 200), seed=95, max_kv_len=200)
    _check(w, wl.draw_q_abs(300, 32, seed=96), "300 short sequences")


def test_rows_spanning_decades_one_long_sequence():
    """One 20,000-token sequence in every split, row magnitudes 10^U(-3, 3): the per-row
    exponents vary over 20 binades."""
    w = wl.make_workload(1, 128, [20000], seed=97)
    gen = torch.Generator().manual_seed(98)
    mag = torch.pow(10.0, torch.rand((1, 20000, 1), generator=gen) * 6 - 3)
    w.cache = (w.cache.float() * mag).to(torch.bfloat16)
    _check(w, wl.draw_q_abs(1, 128, seed=99), "decades of row magnitude")


@pytest.mark.parametrize("lo,hi", [(-118, -110), (14, 22), (-20, 20)])
def test_row_exponent_ranges(lo, hi):
    """Row magnitudes 2^U(lo, hi): rows whose expanded values fall below bf16's normal range
    (exponents down to -126), rows past the single-multiply range of the expansion (exponents
    above 7), and both kinds mixed inside every tile."""
    w = wl.make_workload(2, 64, [1000, 333], seed=300 + lo)
    gen = torch.Generator().manual_seed(301 + lo)
    mag = torch.exp2(lo + torch.rand((2, w.cache.shape[1], 1), generator=gen) * (hi - lo))
    w.cache = (w.cache.float() * mag).to(torch.bfloat16)
    _check(w, wl.draw_q_abs(2, 64, seed=102), f"row magnitudes 2^[{lo}, {hi}]")


def test_argument_errors():
    h = binding.MlaDecode(16, 1, 64)
    qa = torch.zeros((1, 16, 576), dtype=torch.bfloat16, device=DEV)
    codes = torch.zeros((1, 64, 576), dtype=torch.uint8, device=DEV)
    lens = torch.tensor([10], dtype=torch.int32, device=DEV)
    with pytest.raises(ValueError):
        h.decode_attn_fp8(qa, codes, torch.zeros((1, 64), dtype=torch.int16, device=DEV), lens)
    with pytest.raises(binding.MlaError, match="INVALID_ARG"):   # a row pitch that is not 16-byte
        wide = torch.zeros((1, 64, 584), dtype=torch.uint8, device=DEV)[..., :576]
        h.decode_attn_fp8(qa, wide, torch.zeros((1, 64), dtype=torch.int8, device=DEV), lens)


@pytest.mark.parametrize("page_size", [0, 64])
def test_cache_write_into_the_quantised_cache(page_size):
    """mla_append_kv_fp8: the new rows' exponents are the oracle's, their codes dequantise to
    within half a step of the oracle's rows, no other row changes, and the decode over the
    quantised cache then matches the oracle over the dequantised rows."""
    lens = [5, 64, 130]
    w = wl.make_workload(3, 32, lens, page_size=page_size, seed=100,
                         max_kv_len=192 if page_size else None)
    g = w.to(DEV)
    codes, exps, _, deq64 = _quantise(w.cache)
    codes, exps = codes.to(DEV), exps.to(DEV)
    before_c, before_e = codes.clone(), exps.clone()
    inp = wl.draw_append_inputs(3, 1024, seed=101)
    h = binding.MlaDecode(32, 3, w.max_kv_len, page_size=page_size)
    dev = {k: v.to(DEV) for k, v in inp.items()}
    h.append_kv_fp8(dev["hidden"], dev["w_dkv"], dev["w_kr"], dev["gamma"], codes, exps, g.kv_lens,
                    g.page_table)
    h.check_device_errors()
    ref = oracle.cache_rows(to_np(inp["hidden"]), to_np(inp["w_dkv"]), to_np(inp["w_kr"]),
                            to_np(inp["gamma"]), lens, w.rope_base)

    def at(b):
        pos = lens[b] - 1
        if w.page_table is None:
            return b, pos
        return int(w.page_table[b, pos // 64]), pos % 64

    mask = torch.ones(codes.shape[:2], dtype=torch.bool, device=DEV)
    for b in range(3):
        i, j = at(b)
        mask[i, j] = False
        e = int(exps[i, j])
        assert e == oracle.fp8_row_exponent(ref[b]), b
        got = oracle.dequantize_rows_fp8(codes[i, j].cpu().numpy()[None], np.array([e]))[0]
        step = 2.0 ** (np.floor(np.log2(np.maximum(np.abs(ref[b]) / 2.0 ** e, 2.0 ** -6))) - 3) * 2.0 ** e
        assert np.all(np.abs(got - ref[b]) <= step / 2 + 1e-6 * np.abs(ref[b]).max()), b
        deq64[i, j] = got
    assert torch.equal(codes[mask], before_c[mask]) and torch.equal(exps[mask], before_e[mask])
    qa = wl.draw_q_abs(3, 32, seed=102)
    lat, lse = h.decode_attn_fp8(qa.to(DEV), codes, exps, g.kv_lens, g.page_table)
    h.check_device_errors()
    a = workload_np(w)
    ref_lat, ref_lse = oracle.latent_attention(to_np(qa), deq64, a["kv_lens"], oracle.default_scale(),
                                               a["page_table"], a["page_size"])
    assert_close(f64(lat), ref_lat, "decode after the quantised cache write: latent")
    assert_close(lse.cpu().numpy(), ref_lse, "decode after the quantised cache write: lse")
