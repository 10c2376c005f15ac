"""Pins of the fp64 oracle to facts the pages and the mathematics fix (CPU only).

Each test is chosen so that a plausible slip in the oracle (a dropped k^R term, a
transposed W_UK, a wrong RoPE sign or frequency, a softmax over the wrong axis, a
page-table index error) fails at least one of them; test_planted_mistakes_are_caught
plants such slips and checks exactly that.
"""

import math
import os

import numpy as np
import pytest
import torch

import oracle
from oracle import mla_oracle as om
from tests import _bruteforce

GOLDEN = os.path.join(os.path.dirname(__file__), "golden", "cache_sizes.txt")


def _golden():
    vals = {}
    with open(GOLDEN) as f:
        for line in f:
            line = line.strip()
            if not line or line.startswith("#"):
                continue
            key, value, tol = line.split()[:3]
            vals[key] = (float(value), float(tol))
    return vals


def _tiny(seed=0, B=2, H=2, d_h=4, d_c=8, d_r=4, L=(5, 3), scale=0.37, base=10.0):
    rng = np.random.default_rng(seed)
    Lmax = max(L)
    return dict(
        q_c=rng.standard_normal((B, H, d_h)), q_r=rng.standard_normal((B, H, d_r)),
        w_uk=rng.standard_normal((H, d_h, d_c)), w_uv=rng.standard_normal((H, d_h, d_c)),
        cache=rng.standard_normal((B, Lmax, d_c + d_r)), kv_lens=np.array(L),
        scale=scale, rope_base=base)


# --- cache arithmetic ------------------------------------------------------------

def test_cache_closed_forms_match_printed_figures():
    g = _golden()
    mha = oracle.mha_cache_elements_per_token(128, 128)
    mla = oracle.mla_cache_elements_per_token(512, 64)

    def close(key, got):
        v, tol = g[key]
        assert abs(got - v) <= tol, (key, got, v)

    close("mha_elements_per_token_per_layer", mha)
    close("mla_elements_per_token_per_layer", mla)
    close("mha_elements_per_token_60_layers", mha * 60)
    close("mla_elements_per_token_60_layers", mla * 60)
    close("mha_over_mla_ratio", mha / mla)
    close("mla_cache_in_units_of_d_h", mla / 128)
    close("mha_bytes_per_token_per_layer_bf16", oracle.kv_cache_bytes(1, 1, mha, 2))
    close("mha_request_bytes_128k_60_layers", oracle.kv_cache_bytes(131072, 60, mha))
    close("mla_request_bytes_128k_60_layers", oracle.kv_cache_bytes(131072, 60, mla))
    # d_c = 4 d_h and d_h^R = d_h / 2 give the 2.25-group GQA equivalence (2 * 2.25 d_h)
    assert mla == 2 * 2.25 * 128


# --- RoPE --------------------------------------------------------------------------

def test_rope_identity_at_position_zero_and_off_switch():
    x = np.random.default_rng(1).standard_normal(64)
    np.testing.assert_array_equal(oracle.rope_rotate(x, 0, 10000.0), x)
    np.testing.assert_array_equal(oracle.rope_rotate(x, 12345, 0.0), x)


def test_rope_matches_complex_product_and_preserves_norm():
    rng = np.random.default_rng(2)
    for pos in (1, 7, 4095, 131071):
        x = rng.standard_normal(64)
        y = oracle.rope_rotate(x, pos, 10000.0)
        z = (x[0::2] + 1j * x[1::2]) * np.exp(1j * pos * 10000.0 ** (-np.arange(32) / 32.0))
        np.testing.assert_allclose(y[0::2], z.real, atol=1e-12)
        np.testing.assert_allclose(y[1::2], z.imag, atol=1e-12)
        assert abs(np.linalg.norm(y) - np.linalg.norm(x)) < 1e-12


def test_rope_first_pair_turns_by_one_radian_per_position():
    # theta_0 = base^0 = 1: position p turns the first pair by p radians; the second pair
    # turns by base^(-2/64) radians per position (10000^(-1/32) = 0.74989420933245...).
    e0 = np.zeros(64)
    e0[0] = 1.0
    y = oracle.rope_rotate(e0, 1, 10000.0)
    assert abs(y[0] - 0.5403023058681398) < 1e-15 and abs(y[1] - 0.8414709848078965) < 1e-15
    e1 = np.zeros(64)
    e1[2] = 1.0
    y = oracle.rope_rotate(e1, 1, 10000.0)
    assert abs(math.atan2(y[3], y[2]) - 0.7498942093324559) < 1e-14


def test_rope_scores_depend_only_on_relative_position():
    rng = np.random.default_rng(3)
    q, k = rng.standard_normal(64), rng.standard_normal(64)
    ref = oracle.rope_rotate(q, 100, 10000.0) @ oracle.rope_rotate(k, 37, 10000.0)
    for shift in (-37, 5, 1000, 50000):
        got = oracle.rope_rotate(q, 100 + shift, 10000.0) @ oracle.rope_rotate(k, 37 + shift, 10000.0)
        assert abs(got - ref) < 1e-9


# --- softmax -----------------------------------------------------------------------

def test_softmax_rows_sum_to_one_shift_invariance_and_lse():
    rng = np.random.default_rng(4)
    s = rng.standard_normal((37, 5)) * 20
    p, lse = oracle.softmax_lse(s, axis=0)
    np.testing.assert_allclose(p.sum(axis=0), 1.0, atol=1e-14)
    p2, lse2 = oracle.softmax_lse(s + 123.0, axis=0)
    np.testing.assert_allclose(p2, p, atol=1e-14)
    np.testing.assert_allclose(lse2, lse + 123.0, atol=1e-12)
    for h in range(5):
        direct = math.log(math.fsum(math.exp(v) for v in s[:, h]))
        assert abs(lse[h] - direct) < 1e-12
    _, lse_empty = oracle.softmax_lse(np.zeros((0, 3)), axis=0)
    assert np.all(np.isneginf(lse_empty))


# --- the decode step -----------------------------------------------------------------

def test_absorbed_equals_nonabsorbed_tiny():
    """The absorption identity q.(W_UK c) = (W_UK^T q).c, through the whole step
    (DeepSeek-V2 walkthrough section 2.3 displayed equation; section 6 check 2)."""
    t = _tiny()
    ref = oracle.mla_decode_nonabsorbed(**t)
    out, latent, lse = oracle.mla_decode_absorbed(**t)
    assert np.max(np.abs(out - ref)) <= 1e-12 * max(1.0, np.max(np.abs(ref)))
    # the latent output, up-projected, is the head output
    np.testing.assert_allclose(oracle.apply_wuv(latent, t["w_uv"]), ref, atol=1e-12)


def test_score_identity_per_token():
    rng = np.random.default_rng(5)
    q = rng.standard_normal(128)
    w = rng.standard_normal((128, 512))
    c = rng.standard_normal(512)
    q_abs = oracle.absorb_query(q[None, None], np.zeros((1, 1, 64)), w[None],
                                np.array([1]), 0.0)[0, 0, :512]
    assert abs(q @ (w @ c) - q_abs @ c) < 1e-10 * np.abs(q).sum() * np.abs(w).max() * 10


def _bruteforce_case(paged):
    rng = np.random.default_rng(6)
    B, H, L = 2, 2, [5, 3]
    q_c = rng.standard_normal((B, H, 128))
    q_r = rng.standard_normal((B, H, 64))
    w_uk = rng.standard_normal((H, 128, 512)) / math.sqrt(512)
    w_uv = rng.standard_normal((H, 128, 512)) / math.sqrt(512)
    logical = [rng.standard_normal((n, 576)) for n in L]
    if not paged:
        cache = np.full((B, max(L), 576), np.nan)
        for b in range(B):
            cache[b, :L[b]] = logical[b]
        pt, ps = None, 0
    else:
        ps = 2
        npages = [(n + ps - 1) // ps for n in L]
        total = sum(npages) + 1
        perm = rng.permutation(total)
        cache = np.full((total, ps, 576), np.nan)
        pt = np.full((B, 3), -1)
        off = 0
        for b in range(B):
            for k in range(npages[b]):
                page = perm[off + k]
                pt[b, k] = page
                for s in range(ps):
                    j = k * ps + s
                    if j < L[b]:
                        cache[page, s] = logical[b][j]
            off += npages[b]
    return q_c, q_r, w_uk, w_uv, cache, np.array(L), pt, ps, logical


@pytest.mark.parametrize("paged", [False, True])
def test_bruteforce_python_loops_agree(paged):
    q_c, q_r, w_uk, w_uv, cache, L, pt, ps, logical = _bruteforce_case(paged)
    scale = 1 / math.sqrt(192)
    ref, ref_lse = _bruteforce.decode(q_c.tolist(), q_r.tolist(), w_uk.tolist(), w_uv.tolist(),
                                      lambda b: logical[b].tolist(), L.tolist(), scale, 10000.0)
    got = oracle.mla_decode_nonabsorbed(q_c, q_r, w_uk, w_uv, cache, L, scale, 10000.0, pt, ps)
    np.testing.assert_allclose(got, np.array(ref), atol=1e-12)
    out, _, lse = oracle.mla_decode_absorbed(q_c, q_r, w_uk, w_uv, cache, L, scale, 10000.0, pt, ps)
    np.testing.assert_allclose(out, np.array(ref), atol=1e-12)
    np.testing.assert_allclose(lse, np.array(ref_lse), atol=1e-12)


def test_one_token_gives_the_up_projected_latent():
    t = _tiny(L=(1, 1))
    out = oracle.mla_decode_nonabsorbed(**t)
    for b in range(2):
        for i in range(2):
            np.testing.assert_allclose(out[b, i], t["w_uv"][i] @ t["cache"][b, 0, :8], atol=1e-13)


def test_zero_query_gives_the_mean_latent():
    t = _tiny()
    t["q_c"][:] = 0.0
    t["q_r"][:] = 0.0
    out = oracle.mla_decode_nonabsorbed(**t)
    for b, L in enumerate(t["kv_lens"]):
        mean_c = t["cache"][b, :L, :8].mean(axis=0)
        for i in range(2):
            np.testing.assert_allclose(out[b, i], t["w_uv"][i] @ mean_c, atol=1e-13)


def _latent(t):
    """The oracle's absorbed stages up to the latent output, on a _tiny case (d_c = 8)."""
    q_abs = oracle.absorb_query(t["q_c"], t["q_r"], t["w_uk"], t["kv_lens"], t["rope_base"])
    return oracle.latent_attention(q_abs, t["cache"], t["kv_lens"], t["scale"], d_latent=8)


def test_latent_of_one_token_is_its_latent_row():
    """One cached row takes probability 1, so the latent output is exactly that row's d_c
    latent values (not its k^R part), whatever the query. This pins latent_attention
    directly: in _tiny W_UV maps 8 latent values to 4, so an error in its null space would
    pass the head-output pins."""
    t = _tiny(L=(1, 1))
    latent, lse = _latent(t)
    for b in range(2):
        for i in range(2):
            np.testing.assert_array_equal(latent[b, i], t["cache"][b, 0, :8])
    assert np.all(np.isfinite(lse))


def test_latent_of_zero_query_is_the_mean_row_and_lse_is_log_l():
    """A zero absorbed query gives every row the score 0: p = 1/L, the latent output is the
    mean of the L latent rows and the log-sum-exp is log L."""
    t = _tiny(L=(5, 3))
    t["q_c"][:] = 0.0
    t["q_r"][:] = 0.0
    latent, lse = _latent(t)
    for b, L in enumerate(t["kv_lens"]):
        for i in range(2):
            np.testing.assert_allclose(latent[b, i], t["cache"][b, :L, :8].mean(axis=0),
                                       rtol=0, atol=1e-14)
            np.testing.assert_allclose(lse[b, i], math.log(L), rtol=0, atol=1e-14)


def test_latent_of_identical_rows_is_that_row():
    """Rows that are all equal give the same latent output for any query and weights."""
    t = _tiny()
    t["cache"][:] = t["cache"][:, :1, :]
    latent, _ = _latent(t)
    for b in range(2):
        for i in range(2):
            np.testing.assert_allclose(latent[b, i], t["cache"][b, 0, :8], rtol=0, atol=1e-13)


def test_identical_rows_make_the_query_irrelevant():
    t = _tiny()
    t["cache"][:] = t["cache"][:, :1, :]
    out = oracle.mla_decode_nonabsorbed(**t)
    for b in range(2):
        for i in range(2):
            np.testing.assert_allclose(out[b, i], t["w_uv"][i] @ t["cache"][b, 0, :8], atol=1e-12)


def test_zero_position_query_ignores_the_rope_key():
    """DeepSeek-V2 walkthrough section 5.2: with the position path zeroed, the output no
    longer depends on the positional key."""
    t = _tiny()
    t["q_r"][:] = 0.0
    a = oracle.mla_decode_nonabsorbed(**t)
    t["cache"][:, :, 8:] = np.random.default_rng(9).standard_normal(t["cache"][:, :, 8:].shape)
    b = oracle.mla_decode_nonabsorbed(**t)
    np.testing.assert_allclose(a, b, atol=1e-14)
    # and with the position path live, the positional key does matter
    t2 = _tiny()
    a2 = oracle.mla_decode_nonabsorbed(**t2)
    # (a per-token change: adding one vector to every k^R shifts all of a head's scores
    # equally, which the softmax ignores)
    t2["cache"][:, :, 8:] += np.random.default_rng(11).standard_normal(t2["cache"][:, :, 8:].shape)
    assert np.max(np.abs(oracle.mla_decode_nonabsorbed(**t2) - a2)) > 1e-3


def test_empty_sequence_and_unread_rows():
    t = _tiny(L=(4, 0))
    t["cache"][0, 4:] = np.nan          # rows past kv_len are never read
    out = oracle.mla_decode_nonabsorbed(**t)
    assert np.all(np.isfinite(out))
    np.testing.assert_array_equal(out[1], 0.0)
    _, latent, lse = oracle.mla_decode_absorbed(**t)
    np.testing.assert_array_equal(latent[1], 0.0)
    assert np.all(np.isneginf(lse[1])) and np.all(np.isfinite(lse[0]))


def test_paged_layout_equals_contiguous():
    q_c, q_r, w_uk, w_uv, cache_p, L, pt, ps, logical = _bruteforce_case(True)
    cache_c = np.full((2, 5, 576), np.nan)
    for b in range(2):
        cache_c[b, :L[b]] = logical[b]
    s = 1 / math.sqrt(192)
    a = oracle.mla_decode_nonabsorbed(q_c, q_r, w_uk, w_uv, cache_p, L, s, 10000.0, pt, ps)
    b = oracle.mla_decode_nonabsorbed(q_c, q_r, w_uk, w_uv, cache_c, L, s, 10000.0)
    np.testing.assert_array_equal(a, b)


def test_scale_gives_unit_variance_scores_on_the_workload_distributions():
    """With the workloads' distributions (weights std 1/sqrt(512), inputs N(0,1)) the
    scaled scores have variance (128*512/512 + 64)/192 = 1."""
    rng = np.random.default_rng(10)
    H, L = 8, 4000
    q_c = rng.standard_normal((1, H, 128))
    q_r = rng.standard_normal((1, H, 64))
    w_uk = rng.standard_normal((H, 128, 512)) / math.sqrt(512)
    cache = rng.standard_normal((1, L, 576))
    q_abs = oracle.absorb_query(q_c, q_r, w_uk, np.array([L]), 10000.0)
    s = (cache[0] @ q_abs[0].T) * oracle.default_scale()
    assert 0.85 < s.var() < 1.15


def test_bf16_widening_is_exact():
    vals = np.array([1.0, -2.5, 3.140625, 2.0 ** -100, -1.5 * 2.0 ** 120], dtype=np.float32)
    bits = (vals.view(np.uint32) >> 16).astype(np.uint16)
    np.testing.assert_array_equal(oracle.widen(bits), vals.astype(np.float64))


# --- the pins above catch plausible slips -------------------------------------------

def test_planted_mistakes_are_caught(monkeypatch):
    """Plant typical slips into the oracle (CPU only) and check that the brute-force
    cross-check notices each one."""
    q_c, q_r, w_uk, w_uv, cache, L, pt, ps, logical = _bruteforce_case(True)
    scale = 1 / math.sqrt(192)
    ref, _ = _bruteforce.decode(q_c.tolist(), q_r.tolist(), w_uk.tolist(), w_uv.tolist(),
                                lambda b: logical[b].tolist(), L.tolist(), scale, 10000.0)
    ref = np.array(ref)
    good_rotate, good_rows = om.rope_rotate, om.token_rows

    def wrong_sign(x, pos, base, yarn=None):
        return good_rotate(x, -pos, base, yarn)

    def off_by_one(x, pos, base, yarn=None):
        return good_rotate(x, pos + 1, base, yarn)

    def wrong_slot(cache, b, kv_len, page_table=None, page_size=0):
        # slot index off by one inside each page (the order of the rows alone would not
        # matter: attention does not depend on the order of its keys)
        j = np.arange(kv_len)
        return om.widen(np.asarray(cache)[np.asarray(page_table)[b, j // page_size],
                                          (j + 1) % page_size, :])

    def no_rope_key(cache, b, kv_len, page_table=None, page_size=0):
        r = good_rows(cache, b, kv_len, page_table, page_size)
        r[:, 512:] = 0.0
        return r

    for name, fn in [("rope_rotate", wrong_sign), ("rope_rotate", off_by_one),
                     ("token_rows", wrong_slot), ("token_rows", no_rope_key)]:
        with monkeypatch.context() as m:
            m.setattr(om, name, fn)
            got = om.mla_decode_nonabsorbed(q_c, q_r, w_uk, w_uv, cache, L, scale, 10000.0, pt, ps)
        assert not np.allclose(got, ref, atol=1e-6), f"planted {fn.__name__} not caught"
    # the two up-projections swapped (W_UK where W_UV belongs)
    got = om.mla_decode_nonabsorbed(q_c, q_r, w_uk, w_uk, cache, L, scale, 10000.0, pt, ps)
    assert not np.allclose(got, ref, atol=1e-6)


# ---------------------------------------------------------------------------
# the cache row of a new token (the step before decode)
# ---------------------------------------------------------------------------

def test_rms_norm_closed_form_unit_rms_and_scale_invariance():
    # [3, 4]: mean square 12.5, so [3, 4] / sqrt(12.5) = [0.8485..., 1.1313...]
    y = oracle.rms_norm(np.array([3.0, 4.0]), np.ones(2), eps=0.0)
    np.testing.assert_allclose(y, [3 / math.sqrt(12.5), 4 / math.sqrt(12.5)], rtol=1e-15)
    rng = np.random.default_rng(40)
    x = rng.standard_normal(512)
    y = oracle.rms_norm(x, np.ones(512), eps=0.0)
    assert abs(np.sqrt(np.mean(y * y)) - 1.0) < 1e-14
    np.testing.assert_allclose(oracle.rms_norm(7.5 * x, np.ones(512), eps=0.0), y, rtol=1e-13)
    g = rng.standard_normal(512)
    np.testing.assert_allclose(oracle.rms_norm(x, g, eps=0.0), y * g, rtol=1e-13)


def _tiny_append(seed=41, d=16, d_c=8, d_r=4, B=3):
    rng = np.random.default_rng(seed)
    h = rng.standard_normal((B, d))
    w_dkv = rng.standard_normal((d_c, d)) / math.sqrt(d)
    w_kr = rng.standard_normal((d_r, d)) / math.sqrt(d)
    gamma = 1.0 + 0.1 * rng.standard_normal(d_c)
    lens = np.array([1, 5, 77])[:B]
    return h, w_dkv, w_kr, gamma, lens


def test_cache_rows_match_python_loops():
    h, w_dkv, w_kr, gamma, lens = _tiny_append()
    got = oracle.cache_rows(h, w_dkv, w_kr, gamma, lens, 10000.0)
    for b in range(len(lens)):
        ref = _bruteforce.cache_row(h[b].tolist(), w_dkv.tolist(), w_kr.tolist(), gamma.tolist(),
                                    int(lens[b]), 10000.0)
        np.testing.assert_allclose(got[b], ref, rtol=1e-12, atol=1e-14)


def test_appended_key_and_query_at_the_same_position_keep_their_dot_product():
    """The new token's k^R is rotated at kv_len-1, the position the decode step rotates the
    query to: their dot product is the unrotated one (rotations by one angle cancel)."""
    rng = np.random.default_rng(42)
    d, d_r = 32, 64
    h = rng.standard_normal((1, d))
    w_kr = rng.standard_normal((d_r, d))
    q_r = rng.standard_normal(d_r)
    for L in (1, 2, 4097, 131072):
        row = oracle.cache_rows(h, np.zeros((8, d)), w_kr, np.ones(8), [L], 10000.0)[0]
        k_rot = row[8:]
        q_rot = oracle.rope_rotate(q_r, L - 1, 10000.0)
        assert abs(q_rot @ k_rot - q_r @ (w_kr @ h[0])) < 1e-9 * (1 + abs(q_r @ (w_kr @ h[0])))


def test_cache_row_planted_mistakes_are_caught():
    h, w_dkv, w_kr, gamma, lens = _tiny_append(seed=43)
    good = oracle.cache_rows(h, w_dkv, w_kr, gamma, lens, 10000.0)
    x = h @ w_dkv.T
    # gamma dropped
    no_gamma = x / np.sqrt(np.mean(x * x, axis=1, keepdims=True) + 1e-6)
    assert np.max(np.abs(no_gamma - good[:, :8])) > 1e-3
    # the norm taken over the whole 576-wide row instead of the latent only
    full = np.concatenate([x, h @ w_kr.T], axis=1)
    whole = full / np.sqrt(np.mean(full * full, axis=1, keepdims=True) + 1e-6)
    assert np.max(np.abs(whole[:, :8] * gamma - good[:, :8])) > 1e-3
    # RoPE one position late (at kv_len instead of kv_len - 1)
    late = np.stack([oracle.rope_rotate(w_kr @ h[b], int(lens[b]), 10000.0) for b in range(len(lens))])
    assert np.max(np.abs(late - good[:, 8:])) > 1e-3


# --- YaRN (context extension of the decoupled RoPE) --------------------------------

YARN_GOLDEN = os.path.join(os.path.dirname(__file__), "golden", "yarn.txt")


def _yarn_golden():
    vals = {}
    with open(YARN_GOLDEN) as f:
        for line in f:
            line = line.strip()
            if line and not line.startswith("#"):
                key, value = line.split()[:2]
                vals[key] = float(value)
    return vals


def _pages_yarn():
    g = _yarn_golden()
    return oracle.Yarn(factor=g["scale_factor_s"], original_len=int(g["original_length_tokens"]),
                       alpha=g["alpha"], beta=g["beta"], mscale_coef=g["sqrt_t_coefficient"])


def test_yarn_figures_are_consistent():
    """The pages' target length is the scale factor times the original 4K context."""
    g = _yarn_golden()
    assert g["scale_factor_s"] * g["original_length_tokens"] == g["target_length_tokens"]


def test_yarn_off_or_factor_one_is_plain_rope():
    plain = oracle.rope_theta(64, 10000.0)
    np.testing.assert_array_equal(oracle.rope_theta(64, 10000.0, None), plain)
    np.testing.assert_allclose(oracle.rope_theta(64, 10000.0, oracle.Yarn(factor=1.0)), plain, rtol=0)
    assert oracle.yarn_score_factor(None) == 1.0
    assert oracle.yarn_score_factor(oracle.Yarn(factor=1.0)) == 1.0


def test_yarn_keeps_fast_pairs_and_slows_slow_pairs_by_s():
    """With the pages' s = 40 over a 4K context: pair 0 (wavelength 2 pi, fits 652 times)
    is kept, pair 31 (wavelength ~47,000 > 4K) is slowed by exactly s, and every pair lies
    between theta/s and theta, non-increasing in m."""
    y = _pages_yarn()
    plain = oracle.rope_theta(64, 10000.0)
    th = oracle.rope_theta(64, 10000.0, y)
    assert th[0] == plain[0]
    np.testing.assert_allclose(th[31], plain[31] / 40.0, rtol=1e-15)
    assert np.all(th <= plain * (1 + 1e-15)) and np.all(th >= plain / 40.0 * (1 - 1e-15))
    assert np.all(np.diff(th) <= 0)
    # some pairs sit on the ramp (neither kept nor fully slowed)
    mid = (th < plain * (1 - 1e-12)) & (th > plain / 40.0 * (1 + 1e-12))
    assert mid.sum() >= 3


def test_yarn_theta_matches_python_loops():
    for y in (_pages_yarn(), oracle.Yarn(factor=8.0, original_len=2048, alpha=2.0, beta=16.0)):
        got = oracle.rope_theta(64, 10000.0, y)
        ref = _bruteforce.yarn_theta(64, 10000.0, y.factor, y.original_len, y.alpha, y.beta)
        np.testing.assert_allclose(got, ref, rtol=1e-14)
        rng = np.random.default_rng(50)
        x = rng.standard_normal(64)
        np.testing.assert_allclose(oracle.rope_rotate(x, 100000, 10000.0, y),
                                   _bruteforce.rotate_with(list(x), 100000, ref), atol=1e-9)


def test_yarn_score_factor_special_points():
    """sqrt(t) = c ln s + 1: t = 1 at s = 1, and t = 4 where c ln s = 1."""
    c = 0.0707
    assert oracle.yarn_score_factor(oracle.Yarn(factor=1.0, mscale_coef=c)) == 1.0
    s = math.exp(1.0 / c)
    assert abs(oracle.yarn_score_factor(oracle.Yarn(factor=s, mscale_coef=c)) - 4.0) < 1e-12
    assert oracle.default_scale(yarn=oracle.Yarn(factor=s, mscale_coef=c)) == pytest.approx(4.0 / math.sqrt(192))


def test_yarn_rotation_keeps_relative_position_property():
    """Rotations with any fixed frequencies: q at p and k at p' give the same dot product as
    q at p + d and k at p' + d."""
    y = _pages_yarn()
    rng = np.random.default_rng(51)
    q, k = rng.standard_normal(64), rng.standard_normal(64)
    a = oracle.rope_rotate(q, 5000, 10000.0, y) @ oracle.rope_rotate(k, 1234, 10000.0, y)
    b = oracle.rope_rotate(q, 105000, 10000.0, y) @ oracle.rope_rotate(k, 101234, 10000.0, y)
    assert abs(a - b) < 1e-9


def test_yarn_planted_mistakes_are_caught():
    y = _pages_yarn()
    plain = oracle.rope_theta(64, 10000.0)
    good = oracle.rope_theta(64, 10000.0, y)
    r = y.original_len * plain / (2 * math.pi)
    g = np.clip((r - y.alpha) / (y.beta - y.alpha), 0, 1)
    reversed_ramp = g * plain / y.factor + (1 - g) * plain
    multiplied = (1 - g) * plain * y.factor + g * plain
    for bad in (reversed_ramp, multiplied):
        assert not np.allclose(bad, good)
        # ... and the pin on the end pairs sees it
        assert bad[0] != plain[0] or abs(bad[31] - plain[31] / 40.0) > 1e-18


# --- several new tokens per sequence (multi-token / speculative decoding) ----------

def _tiny_tokens(seed=60, B=2, T=3, H=2, d_h=4, d_c=8, d_r=4, L=(7, 2)):
    rng = np.random.default_rng(seed)
    Lmax = max(L)
    return dict(q_c=rng.standard_normal((B, T, H, d_h)), q_r=rng.standard_normal((B, T, H, d_r)),
                w_uk=rng.standard_normal((H, d_h, d_c)), w_uv=rng.standard_normal((H, d_h, d_c)),
                cache=rng.standard_normal((B, Lmax, d_c + d_r)), kv_lens=np.array(L))


def test_tokens_with_one_token_equal_single_token_decode():
    a = _tiny_tokens(T=1, L=(7, 3))
    q1 = oracle.absorb_query(a["q_c"][:, 0], a["q_r"][:, 0], a["w_uk"], a["kv_lens"], 10.0)
    qt = oracle.absorb_query_tokens(a["q_c"], a["q_r"], a["w_uk"], a["kv_lens"], 10.0)
    np.testing.assert_array_equal(qt[:, 0], q1)
    l1, s1 = oracle.latent_attention(q1, a["cache"], a["kv_lens"], 0.3, d_latent=8)
    lt, st = oracle.latent_attention_tokens(qt, a["cache"], a["kv_lens"], 0.3, d_latent=8)
    np.testing.assert_allclose(lt[:, 0], l1, rtol=1e-13, atol=1e-13)
    np.testing.assert_allclose(st[:, 0], s1, rtol=1e-13)


def test_each_new_token_is_a_single_token_decode_on_the_truncated_cache():
    """Token t of T over L rows is exactly the one-token decode over the first L - T + t + 1
    rows (its position is the last of them): checked against the pure-Python brute force."""
    a = _tiny_tokens()
    B, T, H = a["q_c"].shape[:3]
    got = oracle.mla_decode_nonabsorbed_tokens(a["q_c"], a["q_r"], a["w_uk"], a["w_uv"], a["cache"],
                                               a["kv_lens"], 0.41, 10.0)
    for b in range(B):
        for t in range(T):
            n = int(a["kv_lens"][b]) - T + t + 1
            if n <= 0:
                np.testing.assert_array_equal(got[b, t], 0.0)
                continue
            out, _ = _bruteforce.decode(
                [a["q_c"][b, t].tolist()], [a["q_r"][b, t].tolist()], a["w_uk"].tolist(),
                a["w_uv"].tolist(), lambda _b, b=b, n=n: a["cache"][b, :n].tolist(), [n], 0.41, 10.0)
            np.testing.assert_allclose(got[b, t], np.array(out[0]), rtol=1e-12, atol=1e-12)


def test_tokens_absorbed_equals_nonabsorbed():
    a = _tiny_tokens(seed=61, L=(9, 3))
    q = oracle.absorb_query_tokens(a["q_c"], a["q_r"], a["w_uk"], a["kv_lens"], 10.0)
    lat, _ = oracle.latent_attention_tokens(q, a["cache"], a["kv_lens"], 0.41, d_latent=8)
    out_abs = np.einsum("btic,idc->btid", lat, a["w_uv"])
    out = oracle.mla_decode_nonabsorbed_tokens(a["q_c"], a["q_r"], a["w_uk"], a["w_uv"], a["cache"],
                                               a["kv_lens"], 0.41, 10.0)
    np.testing.assert_allclose(out_abs, out, rtol=1e-11, atol=1e-12)


def test_new_tokens_do_not_see_later_new_tokens():
    a = _tiny_tokens(seed=62, L=(9, 5))
    q = oracle.absorb_query_tokens(a["q_c"], a["q_r"], a["w_uk"], a["kv_lens"], 10.0)
    base, _ = oracle.latent_attention_tokens(q, a["cache"], a["kv_lens"], 0.41, d_latent=8)
    changed = a["cache"].copy()
    changed[0, 8] += 5.0          # the last new token of sequence 0 (position 8 of 9)
    lat, _ = oracle.latent_attention_tokens(q, changed, a["kv_lens"], 0.41, d_latent=8)
    np.testing.assert_array_equal(lat[0, :2], base[0, :2])   # tokens 0 and 1 do not see it
    assert not np.allclose(lat[0, 2], base[0, 2])            # token 2 (itself) does
    np.testing.assert_array_equal(lat[1], base[1])


def test_tokens_without_visible_rows():
    a = _tiny_tokens(seed=63, T=3, L=(1, 0))
    q = oracle.absorb_query_tokens(a["q_c"], a["q_r"], a["w_uk"], a["kv_lens"], 10.0)
    lat, lse = oracle.latent_attention_tokens(q, a["cache"], a["kv_lens"], 0.41, d_latent=8)
    assert np.all(lat[0, :2] == 0) and np.all(np.isneginf(lse[0, :2]))
    assert np.all(np.isfinite(lse[0, 2]))
    assert np.all(lat[1] == 0) and np.all(np.isneginf(lse[1]))


# --- the quantised latent cache (E4M3 rows, one power-of-two scale per token) ------------

def test_e4m3_values_at_defining_codes():
    v = oracle.e4m3_value
    assert v(0x00) == 0.0 and math.copysign(1.0, v(0x80)) == -1.0
    assert v(0x01) == 2.0 ** -9          # smallest subnormal
    assert v(0x08) == 2.0 ** -6          # smallest normal
    assert v(0x38) == 1.0
    assert v(0x7E) == 448.0 and v(0xFE) == -448.0
    assert math.isnan(v(0x7F)) and math.isnan(v(0xFF))


def test_e4m3_matches_torch_float8_cast():
    """Every code decodes as torch's float8_e4m3fn does, and round-to-nearest-even encoding of
    random values agrees with torch's cast (both the library routine and the definition)."""
    codes = torch.arange(256, dtype=torch.uint8)
    ref = codes.view(torch.float8_e4m3fn).to(torch.float64).numpy()
    got = oracle.e4m3_decode(codes.numpy())
    assert np.array_equal(np.isnan(ref), np.isnan(got))
    assert np.array_equal(ref[~np.isnan(ref)], got[~np.isnan(got)])
    rng = np.random.default_rng(90)
    x = np.concatenate([rng.uniform(-448, 448, 4000), rng.standard_normal(4000) * 0.01,
                        rng.standard_normal(2000) * 2.0 ** -8])
    ours = oracle.e4m3_encode(x)
    theirs = torch.from_numpy(x).to(torch.float32).to(torch.float8_e4m3fn).view(torch.uint8).numpy()
    assert np.array_equal(ours, theirs)


def test_fp8_rows_quantise_within_half_a_step():
    rng = np.random.default_rng(91)
    rows = rng.standard_normal((20, 576)) * np.exp(rng.uniform(-8, 8, (20, 1)))
    rows[3] = 0.0
    codes, exps = oracle.quantize_rows_fp8(rows)
    deq = oracle.dequantize_rows_fp8(codes, exps)
    for r, e, d in zip(rows, exps, deq):
        amax = np.max(np.abs(r))
        if amax == 0:
            assert np.all(d == 0)
            continue
        assert 224.0 < amax / 2.0 ** e <= 448.0          # the smallest exponent that fits
        step = 2.0 ** (np.floor(np.log2(np.maximum(np.abs(r) / 2.0 ** e, 2.0 ** -6))) - 3) * 2.0 ** e
        assert np.all(np.abs(d - r) <= step / 2 * (1 + 1e-12))


def test_fp8_weight_tiles_have_their_own_scale_and_dequantise_within_half_a_step():
    """FP8 weights: one power-of-two scale per 1 x 128 tile of a weight row (DeepSeek-V3
    walkthrough, section 4.4). A tile's exponent depends on its own 128 values only (a row
    with one large tile keeps its small tiles' resolution), and the dequantised weight is
    within half an E4M3 step of the original everywhere."""
    rng = np.random.default_rng(92)
    w = rng.standard_normal((2, 4, 512)) / math.sqrt(512)      # 2 heads of d_h = 4 rows
    w[0, 1, 128:256] *= 1000.0                                   # one large tile in row 1
    codes, exps = oracle.quantize_weight_fp8(w)
    assert codes.shape == (8, 512) and exps.shape == (8, 4)
    rows = w.reshape(8, 512)
    for r in range(8):
        for t in range(4):
            tile = rows[r, 128 * t:128 * (t + 1)]
            assert exps[r, t] == oracle.fp8_row_exponent(tile)
    assert exps[1, 1] - exps[1, 0] >= 9                          # the large tile's own scale
    deq = oracle.dequantize_weight_fp8(codes, exps, d_head=4)
    assert deq.shape == (2, 4, 512)
    full = deq.reshape(8, 512)
    for r in range(8):
        for t in range(4):
            e = exps[r, t]
            x = rows[r, 128 * t:128 * (t + 1)]
            step = 2.0 ** (np.floor(np.log2(np.maximum(np.abs(x) / 2.0 ** e, 2.0 ** -6))) - 3) * 2.0 ** e
            assert np.all(np.abs(full[r, 128 * t:128 * (t + 1)] - x) <= step / 2 * (1 + 1e-12))
    # the codes decode to exactly value(code) * 2^e: a table lookup of the E4M3 definition
    assert full[0, 0] == oracle.e4m3_value(int(codes[0, 0])) * 2.0 ** exps[0, 0]
