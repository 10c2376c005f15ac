"""The seeded input generators: deterministic, shaped as the workloads say, with every
row that is not part of a sequence poisoned with NaN (CPU only)."""

import torch

from mla_latent_kv_28_b200 import workloads as wl


def test_same_seed_same_inputs_other_seed_other_inputs():
    a = wl.make_workload(2, 4, [7, 3], page_size=4, seed=3)
    b = wl.make_workload(2, 4, [7, 3], page_size=4, seed=3)
    c = wl.make_workload(2, 4, [7, 3], page_size=4, seed=4)
    for name in ("q_c", "q_r", "w_uk", "w_uv", "cache", "page_table", "kv_lens"):
        x, y = getattr(a, name), getattr(b, name)
        assert torch.equal(x.view(torch.int16) if x.is_floating_point() else x,
                           y.view(torch.int16) if y.is_floating_point() else y), name
    assert not torch.equal(a.q_c, c.q_c)


def test_contiguous_shapes_and_poisoned_tail():
    w = wl.make_workload(3, 2, [5, 1, 8], rope_base=10000.0)
    assert w.cache.shape == (3, 8, 576) and w.cache.dtype == torch.bfloat16
    assert w.q_c.shape == (3, 2, 128) and w.q_r.shape == (3, 2, 64)
    assert w.w_uk.shape == (2, 128, 512) and w.w_uv.shape == (2, 128, 512)
    for b, L in enumerate([5, 1, 8]):
        assert torch.isfinite(w.cache[b, :L].float()).all()
        assert torch.isnan(w.cache[b, L:].float()).all()


def test_paged_table_is_a_partial_permutation_with_poisoned_tails():
    w = wl.make_workload(4, 2, [130, 64, 1, 0], page_size=64, spare_pages=5, max_kv_len=256)
    pt = w.page_table
    assert pt.shape == (4, 4)
    used = [int(p) for row in pt for p in row if p >= 0]
    assert len(used) == len(set(used)) == 3 + 1 + 1 + 0
    assert w.num_pages == len(used) + 5
    for b, L in enumerate([130, 64, 1, 0]):
        n = (L + 63) // 64
        assert (pt[b, :n] >= 0).all() and (pt[b, n:] == -1).all()
        for j in range(L):
            assert torch.isfinite(w.cache[int(pt[b, j // 64]), j % 64].float()).all()
        if n and L % 64:
            assert torch.isnan(w.cache[int(pt[b, n - 1]), L % 64:].float()).all()
    spare = sorted(set(range(w.num_pages)) - set(used))
    assert torch.isnan(w.cache[spare].float()).all()


def test_uniform_lengths_in_range_and_lognormal_scales():
    w = wl.make_workload(64, 1, ("uniform", 1, 16384), page_size=64, max_kv_len=16384)
    assert int(w.kv_lens.min()) >= 1 and int(w.kv_lens.max()) <= 16384
    assert len(set(w.kv_lens.tolist())) > 50
    ln = wl.make_workload(1, 1, 4096, latent_scale="lognormal")
    rms = ln.cache[0, :, :512].float().pow(2).mean(dim=1).sqrt()
    # LogNormal(0, 0.5) per-token scales: log-rms has std near 0.5
    assert 0.4 < float(rms.log().std()) < 0.6
    kr = ln.cache[0, :, 512:].float()
    assert 0.9 < float(kr.std()) < 1.1


def test_weight_scale_is_one_over_sqrt_fan_in():
    w = wl.make_workload(1, 8, 16)
    std = float(w.w_uk.float().std())
    assert abs(std - 512 ** -0.5) < 0.002


def test_named_configs_exist():
    assert set(wl.CONFIGS) == {"tiny_h16_l256", "v2_b32_l4096", "long_b4_l32768",
                               "single_l131072_lognormal", "ragged_paged_b64"}
    w = wl.config_workload("tiny_h16_l256")
    assert w.batch == 1 and w.n_heads == 16 and int(w.kv_lens[0]) == 256 and w.rope_base == 0.0
