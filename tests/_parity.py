"""Helpers for the GPU parity tests: the tolerance, tensor conversion, oracle calls."""

import numpy as np
import torch

import oracle

# Floating-point bar for every bf16 output against the fp64 oracle:
# max|d| <= 1e-2 * max|ref| and relative L2 error <= 5e-3.
MAX_REL = 1e-2
L2_REL = 5e-3


def to_np(t: torch.Tensor) -> np.ndarray:
    """bf16 / fp32 torch tensor -> numpy (bf16 kept as uint16 bit patterns, which the
    oracle widens exactly)."""
    t = t.detach().cpu()
    if t.dtype == torch.bfloat16:
        return t.view(torch.int16).numpy().view(np.uint16)
    return t.numpy()


def f64(t: torch.Tensor) -> np.ndarray:
    return oracle.widen(to_np(t))


def errors(got, ref):
    got = np.asarray(got, dtype=np.float64)
    ref = np.asarray(ref, dtype=np.float64)
    d = got - ref
    max_ref = float(np.max(np.abs(ref))) if ref.size else 0.0
    return float(np.max(np.abs(d))) if d.size else 0.0, max_ref, \
        float(np.linalg.norm(d) / max(np.linalg.norm(ref), 1e-300))


def assert_close(got, ref, what: str):
    got = np.asarray(got, dtype=np.float64)
    ref = np.asarray(ref, dtype=np.float64)
    assert got.shape == ref.shape, (what, got.shape, ref.shape)
    assert np.all(np.isfinite(got)), f"{what}: non-finite values"
    if not np.any(ref):
        assert np.all(got == 0), f"{what}: expected exact zeros"
        return
    max_err, max_ref, l2 = errors(got, ref)
    assert max_err <= MAX_REL * max_ref, f"{what}: max|d| {max_err:.3e} > 1e-2 * {max_ref:.3e}"
    assert l2 <= L2_REL, f"{what}: rel-L2 {l2:.3e} > 5e-3"


def workload_np(w):
    """The workload's inputs as numpy (bf16 bit patterns) for the oracle."""
    return dict(q_c=to_np(w.q_c), q_r=to_np(w.q_r), w_uk=to_np(w.w_uk), w_uv=to_np(w.w_uv),
                cache=to_np(w.cache), kv_lens=w.kv_lens.cpu().numpy(),
                page_table=None if w.page_table is None else w.page_table.cpu().numpy(),
                page_size=w.page_size)


def quantise_weight_e4m3(w: torch.Tensor):
    """Test input preparation: a bf16 weight [n_h, 128, 512] as E4M3 codes [n_h * 128, 512]
    and one power-of-two exponent per 1 x 128 tile [n_h * 128, 4] (the smallest e with
    max|tile| / 2^e <= 448; codes by torch's float8_e4m3fn cast, round to nearest even).
    tests/test_gpu_fp8_weights.py checks both against the oracle's quantiser on samples."""
    rows = w.detach().cpu().double().reshape(-1, 4, 128)
    amax = rows.abs().amax(dim=2)
    e = torch.where(amax > 0, torch.ceil(torch.log2(amax / 448.0)), torch.zeros_like(amax))
    e = e + (amax / torch.exp2(e) > 448.0).double()
    e = e - ((amax > 0) & (amax / torch.exp2(e - 1) <= 448.0)).double()
    codes = (rows / torch.exp2(e)[:, :, None]).float().to(torch.float8_e4m3fn).view(torch.uint8)
    return codes.reshape(-1, 512).contiguous(), e.to(torch.int8).contiguous()
