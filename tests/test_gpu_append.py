"""GPU parity of the cache write (mla_append_kv) against the fp64 oracle: the row written for
each sequence's new token, element by element, every other cache row left bit for bit as it
was, the contiguous and the paged layout, hidden sizes from one 64-column box to the largest
supported, batches over one tile of sequences, the device error bits, and the composition
with the decode attention that reads the row back."""

import numpy as np
import pytest
import torch

import oracle
from mla_latent_kv_28_b200 import binding
from mla_latent_kv_28_b200 import workloads as wl
from tests._parity import assert_close, f64, to_np, workload_np

pytestmark = pytest.mark.gpu

DEV = "cuda:0"


def _row_index(w, b):
    """(first index, second index) of token kv_len[b]-1 of sequence b in w.cache."""
    pos = int(w.kv_lens[b]) - 1
    if w.page_table is None:
        return b, pos
    return int(w.page_table[b, pos // w.page_size]), pos % w.page_size


def _append_and_check(w, d_model, seed, what, eps=1e-6):
    inp = wl.draw_append_inputs(w.batch, d_model, seed=seed)
    g = w.to(DEV)
    before = g.cache.clone()
    h = binding.MlaDecode(w.n_heads, w.batch, w.max_kv_len, page_size=w.page_size,
                          rope_base=w.rope_base)
    dev = {k: v.to(DEV) for k, v in inp.items()}
    h.append_kv(dev["hidden"], dev["w_dkv"], dev["w_kr"], dev["gamma"], g.cache, g.kv_lens,
                g.page_table, eps=eps)
    h.check_device_errors()
    ref = oracle.cache_rows(to_np(inp["hidden"]), to_np(inp["w_dkv"]), to_np(inp["w_kr"]),
                            to_np(inp["gamma"]), w.kv_lens.numpy(), w.rope_base, eps)
    got = np.stack([f64(g.cache[_row_index(w, b)]) for b in range(w.batch)])
    assert_close(got[:, :512], ref[:, :512], f"{what}: c^KV rows")
    assert_close(got[:, 512:], ref[:, 512:], f"{what}: k^R rows")
    # every other row is untouched (bit patterns, so the NaN fill compares too)
    mask = torch.ones(g.cache.shape[:2], dtype=torch.bool, device=DEV)
    for b in range(w.batch):
        mask[_row_index(w, b)] = False
    assert torch.equal(g.cache.view(torch.int16)[mask], before.view(torch.int16)[mask]), \
        f"{what}: a row other than the new tokens' changed"
    return h, g, ref


def test_contiguous_full_size():
    """Batch 32 at DeepSeek-V2's hidden size 5120: 16 slices of 320 columns."""
    w = wl.make_workload(32, 16, ("uniform", 1, 700), seed=41)
    _append_and_check(w, 5120, 42, "B=32 d=5120 contiguous")


def test_paged_over_one_sequence_tile():
    """70 ragged sequences in 64-token pages: two tiles of sequences in the projection, rows
    landing anywhere in a page (first, last, middle)."""
    w = wl.make_workload(70, 16, ("uniform", 1, 300), page_size=64, seed=43, max_kv_len=300)
    _append_and_check(w, 512, 44, "B=70 d=512 paged")


@pytest.mark.parametrize("d_model", [64, 7168, 8192])
def test_hidden_sizes(d_model):
    """One box in one slice (64), 7 boxes per slice (7168, DeepSeek-V3's size), the largest
    (8192, 8 boxes per slice)."""
    w = wl.make_workload(3, 16, [1, 64, 129], seed=45)
    _append_and_check(w, d_model, 46, f"d={d_model}")


def test_rope_off_and_eps():
    """rope_base 0 leaves k^R as projected; a large eps changes the normalisation."""
    w = wl.make_workload(5, 16, [9, 10, 11, 12, 13], seed=47, rope_base=0.0)
    _append_and_check(w, 1024, 48, "rope off, eps 0.5", eps=0.5)


def test_large_activations():
    """Hidden states 100x the recipe: the RMSNorm must cancel the scale."""
    w = wl.make_workload(4, 16, [100, 200, 300, 400], seed=49)
    inp = wl.draw_append_inputs(4, 2048, seed=50)
    g = w.to(DEV)
    hid = (inp["hidden"].float() * 100).to(torch.bfloat16)
    h = binding.MlaDecode(16, 4, w.max_kv_len, rope_base=w.rope_base)
    h.append_kv(hid.to(DEV), inp["w_dkv"].to(DEV), inp["w_kr"].to(DEV), inp["gamma"].to(DEV),
                g.cache, g.kv_lens)
    h.check_device_errors()
    ref = oracle.cache_rows(to_np(hid), to_np(inp["w_dkv"]), to_np(inp["w_kr"]),
                            to_np(inp["gamma"]), w.kv_lens.numpy(), w.rope_base)
    got = np.stack([f64(g.cache[b, int(w.kv_lens[b]) - 1]) for b in range(4)])
    assert_close(got[:, :512], ref[:, :512], "x100 hidden: c^KV")
    assert_close(got[:, 512:], ref[:, 512:], "x100 hidden: k^R")


def test_append_then_decode():
    """The written rows are where the decode attention reads them: attention over the GPU's
    cache equals the oracle's attention over the oracle's cache with the oracle's rows."""
    w = wl.make_workload(6, 32, ("uniform", 1, 500), page_size=64, seed=51, max_kv_len=500)
    h, g, ref = _append_and_check(w, 5120, 52, "append before decode")
    qa = wl.draw_q_abs(6, 32, seed=53)
    latent, lse = h.decode_attn(qa.to(DEV), g.cache, g.kv_lens, g.page_table)
    h.check_device_errors()
    a = workload_np(w)
    cache64 = oracle.widen(a["cache"]).copy()
    for b in range(w.batch):
        cache64[_row_index(w, b)] = ref[b]
    ref_lat, ref_lse = oracle.latent_attention(to_np(qa), cache64, a["kv_lens"],
                                               oracle.default_scale(), a["page_table"],
                                               a["page_size"])
    assert_close(f64(latent), ref_lat, "decode after append: latent")
    assert_close(lse.cpu().numpy(), ref_lse, "decode after append: lse")


def test_bad_kv_len_and_page_set_error_bits():
    """kv_len 0 (no row to write) sets bit 2; a page id outside the pool sets bit 0. Neither
    sequence's cache is written, the valid one is."""
    w = wl.make_workload(3, 16, [5, 70, 7], page_size=64, seed=54, max_kv_len=128)
    g = w.to(DEV)
    inp = {k: v.to(DEV) for k, v in wl.draw_append_inputs(3, 256, seed=55).items()}
    h = binding.MlaDecode(16, 3, 128, page_size=64)
    lens = g.kv_lens.clone()
    lens[0] = 0
    table = g.page_table.clone()
    table[1, 1] = g.cache.shape[0] + 5      # sequence 1's new token lies in its second page
    before = g.cache.clone()
    h.append_kv(inp["hidden"], inp["w_dkv"], inp["w_kr"], inp["gamma"], g.cache, lens, table)
    with pytest.raises(binding.MlaError) as e:
        h.check_device_errors()
    assert e.value.detail == 0b101
    changed = (g.cache.view(torch.int16) != before.view(torch.int16)).any(dim=-1)
    assert int(changed.sum()) == 1 and bool(changed[_row_index(w, 2)])
    h.check_device_errors()   # the word was cleared by the read


def test_argument_errors():
    w = wl.make_workload(2, 16, [4, 4], seed=56)
    g = w.to(DEV)
    inp = {k: v.to(DEV) for k, v in wl.draw_append_inputs(2, 128, seed=57).items()}
    h = binding.MlaDecode(16, 2, 4)
    args = (inp["hidden"], inp["w_dkv"], inp["w_kr"], inp["gamma"], g.cache, g.kv_lens)
    with pytest.raises(binding.MlaError, match="INVALID_ARG"):
        h.append_kv(*args, eps=-1.0)
    with pytest.raises(binding.MlaError, match="INVALID_ARG"):
        h.append_kv(inp["hidden"][:, :96].contiguous(), inp["w_dkv"][:, :96].contiguous(),
                    inp["w_kr"][:, :96].contiguous(), inp["gamma"], g.cache, g.kv_lens)
    big = torch.zeros((2, 8256), dtype=torch.bfloat16, device=DEV)
    wbig = torch.zeros((512, 8256), dtype=torch.bfloat16, device=DEV)
    with pytest.raises(binding.MlaError, match="UNSUPPORTED"):
        h.append_kv(big, wbig, wbig[:64], inp["gamma"], g.cache, g.kv_lens)
    with pytest.raises(binding.MlaError, match="INVALID_ARG"):   # page table on a contiguous handle
        h.append_kv(*args, page_table=torch.zeros((2, 1), dtype=torch.int32, device=DEV))
    h.check_device_errors()
