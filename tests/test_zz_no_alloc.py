"""mla_decode_attn_noalloc, the handle-free attention call for callers that cannot allocate
device memory (a serving engine whose KV-cache pool owns nearly all of HBM, a plugin host
that forbids cudaMalloc, a hot path that cannot afford cudaMalloc's synchronisation).

Its scratch is a fixed array inside the library, shared by every call, so this checks two
calls in a row of different shapes (the second must not see the first's leftovers) against
the handle-based mla_decode_attn on the same inputs and against the fp64 oracle, within the
tolerance the parity tests use. It also checks the routing of the device error word (the
caller's word, or the library's own when the caller passes none) and a call without lse.
Kept in a file of its own that pytest collects last; it passes alone in a fresh process and
after the other tests.
"""

import ctypes

import pytest
import torch

import oracle
from mla_latent_kv_28_b200 import binding
from mla_latent_kv_28_b200 import workloads as wl
from tests._parity import assert_close, f64, to_np, workload_np

pytestmark = pytest.mark.gpu

DEV = "cuda:0"
ERR_BAD_KV_LEN = 1 << 2   # device error word bit: a kv_len outside 0..max_kv_len


def _noalloc(w, q_abs, err, kv_lens=None, with_lse=True):
    lib = binding.load_library()
    B, H = q_abs.shape[0], q_abs.shape[1]
    out = torch.full((B, H, 512), float("nan"), dtype=torch.bfloat16, device=DEV)
    lse = torch.full((B, H), float("nan"), dtype=torch.float32, device=DEV) if with_lse else None
    cache = w.cache
    row_stride = cache.stride(1)
    paged = w.page_table is not None
    lens = w.kv_lens if kv_lens is None else kv_lens
    st = lib.mla_decode_attn_noalloc(
        H, 0.0, w.page_size, w.max_kv_len, B, q_abs.data_ptr(), cache.data_ptr(),
        cache.data_ptr() + 1024, row_stride, 0 if paged else cache.stride(0) // row_stride,
        lens.data_ptr(), w.page_table.data_ptr() if paged else None,
        w.page_table.shape[1] if paged else 0, cache.shape[0] if paged else 0,
        out.data_ptr(), None if lse is None else lse.data_ptr(),
        None if err is None else err.data_ptr(),
        ctypes.c_void_p(torch.cuda.current_stream().cuda_stream))
    assert st == binding.MLA_OK, binding.load_library().mla_status_string(st)
    return out, lse


def _with_handle(w, q_abs):
    h = binding.MlaDecode(w.n_heads, w.batch, w.max_kv_len, page_size=w.page_size,
                          rope_base=w.rope_base)
    out, lse = h.decode_attn(q_abs, w.cache, w.kv_lens, w.page_table)
    h.check_device_errors()
    h.close()
    return out, lse


def test_two_calls_in_a_row_match_the_handle_path_and_the_oracle():
    first = wl.make_workload(4, 128, [3000, 65, 1, 700], seed=21)
    second = wl.make_workload(9, 64, [1, 64, 129, 2000, 17, 333, 4096, 5, 640], page_size=64,
                              seed=22, max_kv_len=4096)
    err = torch.full((1,), 0xFFFF, dtype=torch.int32, device=DEV)  # the call must clear it
    for w_host in (first, second):
        w = w_host.to(DEV)
        q_host = wl.draw_q_abs(w.batch, w.n_heads, seed=23)
        q_abs = q_host.to(DEV)
        got, got_lse = _noalloc(w, q_abs, err)
        torch.cuda.synchronize()
        assert int(err.item()) == 0, f"device error word {int(err.item()):#x}"
        ref, ref_lse = _with_handle(w, q_abs)
        assert_close(f64(got), f64(ref), f"no-alloc latent ({w.batch} seqs) vs the handle path")
        assert_close(got_lse.cpu().numpy(), ref_lse.cpu().numpy(), "no-alloc lse vs the handle path")
        a = workload_np(w_host)
        o_lat, o_lse = oracle.latent_attention(to_np(q_host), a["cache"], a["kv_lens"],
                                               oracle.default_scale(), a["page_table"],
                                               a["page_size"])
        assert_close(f64(got), o_lat, f"no-alloc latent ({w.batch} seqs) vs the oracle")
        assert_close(got_lse.cpu().numpy(), o_lse, "no-alloc lse vs the oracle")


def test_error_word_routing_and_no_lse():
    w = wl.make_workload(2, 32, [100, 100], seed=26).to(DEV)
    q_abs = wl.draw_q_abs(2, 32, seed=27).to(DEV)
    ref, _ = _with_handle(w, q_abs)
    # a kv_len above max_kv_len is clamped to it by the plan (no read past the cache) and
    # flagged in the caller's error word
    too_long = torch.tensor([100, 101], dtype=torch.int32, device=DEV)
    err = torch.zeros((1,), dtype=torch.int32, device=DEV)
    got, _ = _noalloc(w, q_abs, err, kv_lens=too_long)
    torch.cuda.synchronize()
    assert int(err.item()) & ERR_BAD_KV_LEN, f"device error word {int(err.item()):#x}"
    assert_close(f64(got), f64(ref), "no-alloc latent with a clamped kv_len")
    # no error word of the caller's (the library's own is used) and no lse
    got2, _ = _noalloc(w, q_abs, None, with_lse=False)
    torch.cuda.synchronize()
    assert_close(f64(got2), f64(ref), "no-alloc latent without err_word and lse")


def test_sizes_beyond_the_scratch_limit_are_rejected():
    lib = binding.load_library()
    w = wl.make_workload(65, 8, 4, seed=24).to(DEV)
    q_abs = wl.draw_q_abs(65, 8).to(DEV)
    out = torch.empty((65, 8, 512), dtype=torch.bfloat16, device=DEV)
    st = lib.mla_decode_attn_noalloc(8, 0.0, 0, 4, 65, q_abs.data_ptr(), w.cache.data_ptr(),
                                     w.cache.data_ptr() + 1024, 576, 4, w.kv_lens.data_ptr(), None,
                                     0, 0, out.data_ptr(), None, None, None)
    assert st == binding.MLA_ERR_UNSUPPORTED
