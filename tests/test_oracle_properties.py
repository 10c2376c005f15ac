"""Property checks of the oracle on random small shapes (hypothesis): the numpy oracle against
the pure-Python brute force for one and several new tokens, paged against contiguous, the
absorbed stages against the non-absorbed definition, and the quantised format's round trip."""

import math

import numpy as np
from hypothesis import given, settings, strategies as st

import oracle
from tests import _bruteforce


@st.composite
def small_problem(draw):
    B = draw(st.integers(1, 2))
    H = draw(st.integers(1, 3))
    d_h = draw(st.sampled_from([2, 4]))
    d_c = draw(st.sampled_from([4, 8]))
    d_r = draw(st.sampled_from([2, 4]))
    lens = draw(st.lists(st.integers(0, 6), min_size=B, max_size=B))
    seed = draw(st.integers(0, 2 ** 31 - 1))
    base = draw(st.sampled_from([0.0, 10.0, 10000.0]))
    scale = draw(st.floats(0.05, 1.0))
    rng = np.random.default_rng(seed)
    Lmax = max(1, max(lens))
    return dict(q_c=rng.standard_normal((B, H, d_h)), q_r=rng.standard_normal((B, H, d_r)),
                w_uk=rng.standard_normal((H, d_h, d_c)), w_uv=rng.standard_normal((H, d_h, d_c)),
                cache=rng.standard_normal((B, Lmax, d_c + d_r)), kv_lens=np.array(lens),
                scale=scale, base=base, d_c=d_c)


@settings(max_examples=40, deadline=None)
@given(small_problem())
def test_oracle_equals_brute_force(p):
    got = oracle.mla_decode_nonabsorbed(p["q_c"], p["q_r"], p["w_uk"], p["w_uv"], p["cache"],
                                        p["kv_lens"], p["scale"], p["base"])
    ref, _ = _bruteforce.decode(p["q_c"].tolist(), p["q_r"].tolist(), p["w_uk"].tolist(),
                                p["w_uv"].tolist(), lambda b: p["cache"][b].tolist(),
                                p["kv_lens"].tolist(), p["scale"], p["base"])
    np.testing.assert_allclose(got, np.array(ref), rtol=1e-10, atol=1e-10)


@settings(max_examples=40, deadline=None)
@given(small_problem())
def test_absorbed_stages_equal_the_definition(p):
    out, _, _ = oracle.mla_decode_absorbed(p["q_c"], p["q_r"], p["w_uk"], p["w_uv"], p["cache"],
                                           p["kv_lens"], p["scale"], p["base"])
    ref = oracle.mla_decode_nonabsorbed(p["q_c"], p["q_r"], p["w_uk"], p["w_uv"], p["cache"],
                                        p["kv_lens"], p["scale"], p["base"])
    np.testing.assert_allclose(out, ref, rtol=1e-10, atol=1e-11)


@settings(max_examples=40, deadline=None)
@given(small_problem(), st.integers(1, 3))
def test_several_tokens_equal_truncated_single_token_decode(p, T):
    rng = np.random.default_rng(int(p["kv_lens"].sum()) + T)
    B, H, d_h = p["q_c"].shape
    q_c = rng.standard_normal((B, T, H, d_h))
    q_r = rng.standard_normal((B, T, H, p["q_r"].shape[2]))
    got = oracle.mla_decode_nonabsorbed_tokens(q_c, q_r, p["w_uk"], p["w_uv"], p["cache"],
                                               p["kv_lens"], p["scale"], p["base"])
    for b in range(B):
        for t in range(T):
            n = oracle.token_visible_rows(int(p["kv_lens"][b]), T, t)
            one = oracle.mla_decode_nonabsorbed(q_c[b:b + 1, t], q_r[b:b + 1, t], p["w_uk"], p["w_uv"],
                                                p["cache"][b:b + 1], [n], p["scale"], p["base"])
            np.testing.assert_allclose(got[b, t], one[0], rtol=1e-12, atol=1e-12)


@settings(max_examples=40, deadline=None)
@given(st.integers(0, 2 ** 31 - 1), st.floats(-30, 30))
def test_quantised_row_round_trip(seed, log_scale):
    rng = np.random.default_rng(seed)
    row = rng.standard_normal(576) * math.exp(log_scale)
    codes, exps = oracle.quantize_rows_fp8(row[None])
    deq = oracle.dequantize_rows_fp8(codes, exps)[0]
    e = int(exps[0])
    assert 224.0 < np.max(np.abs(row)) / 2.0 ** e <= 448.0
    # every value within half a step of its code (steps of 2^-3 relative in normal range)
    step = 2.0 ** (np.floor(np.log2(np.maximum(np.abs(row) / 2.0 ** e, 2.0 ** -6))) - 3) * 2.0 ** e
    assert np.all(np.abs(deq - row) <= step / 2 * (1 + 1e-12))
