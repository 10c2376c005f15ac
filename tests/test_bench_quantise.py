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


def test_bench_weight_quantiser_matches_the_oracle():
    """The FP8-weight input preparation (1 x 128 tiles) gives the oracle's tile exponents and
    codes: oracle.quantize_weight_fp8 on a small weight, element by element."""
    w = wl.make_workload(1, 2, [4], seed=3).w_uk          # [2, 128, 512] bf16
    codes, exps = bench.quantise_weight_e4m3(w)
    ref_codes, ref_exps = oracle.quantize_weight_fp8(w.float().numpy())
    assert np.array_equal(exps.numpy().astype(np.int64), ref_exps)
    assert np.array_equal(codes.numpy(), ref_codes)
