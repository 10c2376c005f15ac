"""bench.py on the GPU: the JSON line carries every key of the measurement contract."""
import json
import os
import subprocess
import sys

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


@pytest.mark.gpu
def test_bench_json_line():
    r = subprocess.run([sys.executable, os.path.join(ROOT, "bench.py"), "--steps", "5", "--warmup", "3",
                        "--no-cpu-baseline"], capture_output=True, text=True, timeout=600, cwd=ROOT)
    assert r.returncode == 0, r.stderr[-2000:]
    line = json.loads(r.stdout.strip().splitlines()[-1])
    for key in ("metric", "value", "unit", "n_gpus", "steps", "warmup", "ms_per_step", "higher_is_better",
                "scaling", "vs_baseline", "dtype", "data", "config", "roofline", "e2e", "gpu_launches", "clocks"):
        assert key in line, key
    assert line["value"] > 0 and line["e2e"]["value"] > 0 and line["e2e"]["eager_value"] > 0
    assert line["e2e"]["h2d_bytes_per_step"] > 0 and line["e2e"]["d2h_bytes_per_step"] > 0
    roof = line["roofline"]
    assert roof["bound"] == "hbm" and 0 < roof["frac"] < 1.5
    # the headline is the largest single-GPU workload; the other four sit under `workloads`
    assert line["config"]["workload"] == "ragged_paged_b64"
    others = line["workloads"]
    assert sorted(others) == ["long_b4_l32768", "single_l131072_lognormal", "tiny_h16_l256",
                              "v2_b32_l4096"]
    for name, o in others.items():
        assert o["tokens_per_s"] > 0 and o["attn_us"] > 0, name
        assert 0 < o["roofline"]["frac"] < 1.5 and o["e2e"]["value"] > 0, name
        assert o["config"]["workload"] == name
    assert line["gpu_launches"] == 4 * 5
    app = line["append_kv"]
    assert app["us"] > 0 and 0 < app["frac_of_hbm"] < 1.5 and app["gpu_launches"] == 2 * 5
    mt = line["multi_token"]
    assert mt["q_len"] == 8 and mt["attn_us"] > 0 and mt["query_tokens_per_s"] > 0
    hg = line["head_gemms"]
    for k in ("absorb_bf16", "wuv_bf16", "absorb_fp8", "wuv_fp8"):
        assert hg[k]["us"] > 0 and 0 < hg[k]["frac_of_hbm"] < 1.5, k
    assert line["fp8_weights"]["tokens_per_s"] > 0
    pf = line["prefill"]
    assert pf["tokens_per_s"] > 0 and 0 < pf["tensor_frac"] < 1.5
    q8 = line["fp8_cache"]
    assert q8["attn_us"] > 0 and 0 < q8["frac_of_hbm"] < 1.5
