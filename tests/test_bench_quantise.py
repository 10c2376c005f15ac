"""The bench's quantised-cache input preparation gives the oracle's exponents and codes."""
import numpy as np

import bench
import oracle
from mla_latent_kv_28_b200 import workloads as wl


def test_bench_quantiser_matches_the_oracle():
    w = wl.make_workload(3, 16, [70, 5, 130], seed=2, latent_scale="lognormal")
    codes, exps = bench.quantise_cache_e4m3(w.cache)
    rows = w.cache.float().numpy().reshape(-1, 576)
    checked = 0
    for i, r in enumerate(rows):
        if not np.isfinite(r).all():
            assert int(exps.view(-1)[i]) == 0
            continue
        e = oracle.fp8_row_exponent(r)
        assert e == int(exps.view(-1)[i])
        assert np.array_equal(oracle.e4m3_encode(r / 2.0 ** e), codes.view(-1, 576)[i].numpy())
        checked += 1
    assert checked == 70 + 5 + 130
