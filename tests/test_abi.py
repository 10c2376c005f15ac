"""The C-ABI library loads and exports every function include/mla_decode.h declares;
configuration checks and status names work without a GPU (CPU only, no compute calls)."""

import ctypes
import os
import re

import pytest

from mla_latent_kv_28_b200 import binding

HEADER = os.path.join(os.path.dirname(os.path.dirname(__file__)), "include", "mla_decode.h")


def _declared_functions():
    text = open(HEADER).read()
    text = re.sub(r"/\*.*?\*/", "", text, flags=re.S)
    names = re.findall(r"^\s*(?:const\s+)?[A-Za-z_][\w\s\*]*?\b(mla_\w+)\s*\(", text, flags=re.M)
    return sorted(set(names))


@pytest.fixture(scope="module")
def lib():
    if not os.path.exists(binding.LIB_PATH):
        from mla_latent_kv_28_b200 import build
        build.build()
    return binding.load_library()


def test_header_declares_the_five_entry_points():
    names = _declared_functions()
    for n in ("mla_decode_create", "mla_absorb_q", "mla_decode_attn", "mla_apply_wuv", "mla_destroy"):
        assert n in names


def test_library_exports_every_declared_function(lib):
    names = _declared_functions()
    assert names, "no declarations parsed"
    for n in names:
        assert hasattr(lib, n), f"{n} declared in mla_decode.h but not exported"
    assert set(names) <= set(binding.SIGNATURES), "binding is missing a declared function"


def test_status_strings(lib):
    assert lib.mla_status_string(0) == b"MLA_OK"
    assert lib.mla_status_string(-1) == b"MLA_ERR_INVALID_ARG"
    assert lib.mla_status_string(-5) == b"MLA_ERR_DEVICE_CHECK"
    assert lib.mla_status_string(123) == b"MLA_ERR_UNKNOWN"


def test_config_checks(lib):
    ok = binding.make_config(128, 64, 131072)
    assert binding.check_config(ok) == binding.MLA_OK
    assert binding.check_config(binding.make_config(16, 1, 256, rope_base=0.0)) == binding.MLA_OK
    assert binding.check_config(binding.make_config(128, 64, 16384, page_size=64)) == binding.MLA_OK
    bad = [
        (binding.make_config(0, 1, 1), binding.MLA_ERR_INVALID_ARG),
        (binding.make_config(8, 0, 1), binding.MLA_ERR_INVALID_ARG),
        (binding.make_config(8, 1, 0), binding.MLA_ERR_INVALID_ARG),
        (binding.make_config(8, 1, 1, softmax_scale=-1.0), binding.MLA_ERR_INVALID_ARG),
        (binding.make_config(8, 1, 1, max_splits=-2), binding.MLA_ERR_INVALID_ARG),
        (binding.make_config(129, 1, 1), binding.MLA_ERR_UNSUPPORTED),
        (binding.make_config(8, 1, 1, page_size=16), binding.MLA_ERR_UNSUPPORTED),
        (binding.make_config(8, 4096, 1), binding.MLA_ERR_UNSUPPORTED),
        # YaRN: a factor in (0, 1), a ramp that does not rise, a negative coefficient, no
        # original length
        (binding.make_config(8, 1, 1, yarn_factor=0.5), binding.MLA_ERR_INVALID_ARG),
        (binding.make_config(8, 1, 1, yarn_factor=40.0, yarn_alpha=32.0, yarn_beta=32.0),
         binding.MLA_ERR_INVALID_ARG),
        (binding.make_config(8, 1, 1, yarn_factor=40.0, yarn_mscale_coef=-0.1), binding.MLA_ERR_INVALID_ARG),
        (binding.make_config(8, 1, 1, yarn_factor=40.0, yarn_original_len=0), binding.MLA_ERR_INVALID_ARG),
        # several new tokens: at most 2^20 attention rows and 8192 (sequence, token) rows
        (binding.make_config(128, 1, 16, q_len=8193), binding.MLA_ERR_UNSUPPORTED),
        (binding.make_config(16, 512, 16, q_len=17), binding.MLA_ERR_UNSUPPORTED),
        (binding.make_config(16, 1, 16, q_len=-1), binding.MLA_ERR_INVALID_ARG),
    ]
    assert binding.check_config(binding.make_config(16, 128, 4096, q_len=8)) == binding.MLA_OK
    assert binding.check_config(binding.make_config(128, 1, 4096, q_len=4096)) == binding.MLA_OK   # a prefill
    assert binding.check_config(binding.make_config(128, 64, 131072, yarn_factor=40.0)) == binding.MLA_OK
    assert binding.check_config(binding.make_config(8, 1, 1, yarn_factor=1.0)) == binding.MLA_OK
    for cfg, want in bad:
        assert binding.check_config(cfg) == want
    wrong_dims = binding.make_config(8, 1, 1)
    wrong_dims.d_latent = 256
    assert binding.check_config(wrong_dims) == binding.MLA_ERR_UNSUPPORTED
    assert lib.mla_check_config(None) == binding.MLA_ERR_INVALID_ARG


def test_null_handle_and_null_out_are_rejected(lib):
    assert lib.mla_destroy(None) == binding.MLA_OK
    assert lib.mla_decode_create(ctypes.byref(binding.make_config(8, 1, 1)), 0, None) == \
        binding.MLA_ERR_INVALID_ARG
    assert lib.mla_absorb_q(None, 1, None, None, None, None, None, None) == binding.MLA_ERR_INVALID_ARG
    assert lib.mla_decode_attn(None, 1, None, None, None, 576, 1, None, None, 0, 0, None, None,
                               None) == binding.MLA_ERR_INVALID_ARG
    assert lib.mla_apply_wuv(None, 1, None, None, None, None) == binding.MLA_ERR_INVALID_ARG
    assert lib.mla_prefill_attn(None, 1, None, None, None, 576, 1, None, None, 0, 0, None, None,
                                None) == binding.MLA_ERR_INVALID_ARG
    assert lib.mla_absorb_q_fp8(None, 1, None, None, None, None, None, None, None) == binding.MLA_ERR_INVALID_ARG
    assert lib.mla_apply_wuv_fp8(None, 1, None, None, None, None, None) == binding.MLA_ERR_INVALID_ARG
    assert lib.mla_workspace_bytes(None) == -1


def test_library_exports_nothing_but_the_c_abi(lib):
    """Everything but the declared C functions is built with hidden visibility."""
    import shutil
    import subprocess
    nm = shutil.which("nm")
    if nm is None:
        pytest.skip("nm not available")
    out = subprocess.run([nm, "-D", "--defined-only", binding.LIB_PATH], capture_output=True, text=True,
                         check=True).stdout
    exported = {line.split()[-1] for line in out.splitlines() if len(line.split()) == 3 and line.split()[1] == "T"}
    assert exported == set(_declared_functions())
