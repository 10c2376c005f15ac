"""ctypes binding of libmla_decode.so (include/mla_decode.h).

Argument marshalling only: tensors are passed as raw device pointers with their strides,
and every step of the decode path runs in the library's CUDA kernels. torch is used for
device memory and streams. Loading fails loudly if the library has not been built.
"""

from __future__ import annotations

import ctypes
import os
from typing import Optional, Tuple

import torch

LIB_PATH = os.path.join(os.path.dirname(os.path.abspath(__file__)), "libmla_decode.so")

MLA_OK = 0
MLA_ERR_INVALID_ARG = -1
MLA_ERR_UNSUPPORTED = -2
MLA_ERR_CUDA = -3
MLA_ERR_OOM = -4
MLA_ERR_DEVICE_CHECK = -5

ERR_BAD_PAGE = 1 << 0
ERR_TIMEOUT = 1 << 1
ERR_BAD_KV_LEN = 1 << 2

ROW = 576
D_LATENT = 512


class MlaConfig(ctypes.Structure):
    _fields_ = [
        ("n_heads", ctypes.c_int32),
        ("d_head", ctypes.c_int32),
        ("d_latent", ctypes.c_int32),
        ("d_rope", ctypes.c_int32),
        ("page_size", ctypes.c_int32),
        ("max_batch", ctypes.c_int32),
        ("max_kv_len", ctypes.c_int64),
        ("softmax_scale", ctypes.c_float),
        ("rope_base", ctypes.c_float),
        ("max_splits", ctypes.c_int32),
        ("yarn_factor", ctypes.c_float),
        ("yarn_original_len", ctypes.c_int32),
        ("yarn_alpha", ctypes.c_float),
        ("yarn_beta", ctypes.c_float),
        ("yarn_mscale_coef", ctypes.c_float),
        ("q_len", ctypes.c_int32),
    ]


_P = ctypes.c_void_p
_I32 = ctypes.c_int32
_I64 = ctypes.c_int64

# name -> (restype, argtypes); every function include/mla_decode.h declares
SIGNATURES = {
    "mla_check_config": (ctypes.c_int, [ctypes.POINTER(MlaConfig)]),
    "mla_decode_create": (ctypes.c_int, [ctypes.POINTER(MlaConfig), ctypes.c_int, ctypes.POINTER(_P)]),
    "mla_destroy": (ctypes.c_int, [_P]),
    "mla_absorb_q": (ctypes.c_int, [_P, _I32, _P, _P, _P, _P, _P, _P]),
    "mla_decode_attn": (ctypes.c_int, [_P, _I32, _P, _P, _P, _I64, _I64, _P, _P, _I32, _I32, _P, _P, _P]),
    "mla_apply_wuv": (ctypes.c_int, [_P, _I32, _P, _P, _P, _P]),
    "mla_decode_step": (ctypes.c_int, [_P, _I32, _P, _P, _P, _P, _P, _P, _I64, _I64, _P, _P, _I32, _I32,
                                       _P, _P, _P, _P]),
    "mla_prefill_attn": (ctypes.c_int, [_P, _I32, _P, _P, _P, _I64, _I64, _P, _P, _I32, _I32, _P, _P, _P]),
    "mla_absorb_q_fp8": (ctypes.c_int, [_P, _I32, _P, _P, _P, _P, _P, _P, _P]),
    "mla_apply_wuv_fp8": (ctypes.c_int, [_P, _I32, _P, _P, _P, _P, _P]),
    "mla_append_kv_fp8": (ctypes.c_int, [_P, _I32, _I32, _P, _P, _P, _P, ctypes.c_float, _P, _P,
                                         _I64, _I64, _P, _P, _I32, _I32, _P]),
    "mla_decode_attn_fp8": (ctypes.c_int, [_P, _I32, _P, _P, _P, _I64, _I64, _P, _P, _I32, _I32, _P, _P, _P]),
    "mla_decode_attn_partial": (ctypes.c_int, [_P, _I32, _P, _P, _P, _I64, _I64, _P, _P, _I32, _I32,
                                               _P, _P, _P]),
    "mla_merge_partials": (ctypes.c_int, [_P, _I32, _I32, _P, _P, _P, _P, _P]),
    "mla_append_kv": (ctypes.c_int, [_P, _I32, _I32, _P, _P, _P, _P, ctypes.c_float, _P, _P,
                                     _I64, _I64, _P, _P, _I32, _I32, _P]),
    "mla_decode_attn_noalloc": (ctypes.c_int, [_I32, ctypes.c_float, _I32, _I64, _I32, _P, _P, _P,
                                               _I64, _I64, _P, _P, _I32, _I32, _P, _P, _P, _P]),
    "mla_check_device_errors": (ctypes.c_int, [_P, _P, ctypes.POINTER(ctypes.c_uint32)]),
    "mla_workspace_bytes": (ctypes.c_int64, [_P]),
    "mla_status_string": (ctypes.c_char_p, [ctypes.c_int]),
}

_lib = None


def load_library(path: str = LIB_PATH) -> ctypes.CDLL:
    """Load libmla_decode.so once and declare its functions."""
    global _lib
    if _lib is not None:
        return _lib
    if not os.path.exists(path):
        raise RuntimeError(
            f"{path} is missing: build the CUDA library first "
            "(python -m mla_latent_kv_28_b200.build, or __graft_entry__.build())")
    lib = ctypes.CDLL(path)
    for name, (res, args) in SIGNATURES.items():
        fn = getattr(lib, name)
        fn.restype = res
        fn.argtypes = args
    _lib = lib
    return lib


class MlaError(RuntimeError):
    def __init__(self, status: int, what: str, detail: int = 0):
        name = load_library().mla_status_string(status).decode()
        super().__init__(f"{what}: {name} ({status})" + (f", device error word {detail:#x}" if detail else ""))
        self.status = status
        self.detail = detail


def _check(status: int, what: str) -> None:
    if status != MLA_OK:
        raise MlaError(status, what)


def make_config(n_heads: int, max_batch: int, max_kv_len: int, page_size: int = 0,
                softmax_scale: float = 0.0, rope_base: float = 10000.0,
                max_splits: int = 0, yarn_factor: float = 0.0, yarn_original_len: int = 4096,
                yarn_alpha: float = 1.0, yarn_beta: float = 32.0,
                yarn_mscale_coef: float = 0.0707, q_len: int = 1) -> MlaConfig:
    """yarn_factor > 1 turns on YaRN (DeepSeek-V2 uses 40 with the other defaults); q_len > 1
    makes every call take q_len new tokens per sequence (a token axis after the batch axis)."""
    return MlaConfig(n_heads, 128, 512, 64, page_size, max_batch, max_kv_len,
                     softmax_scale, rope_base, max_splits, yarn_factor, yarn_original_len,
                     yarn_alpha, yarn_beta, yarn_mscale_coef, q_len)


def check_config(cfg: MlaConfig) -> int:
    return load_library().mla_check_config(ctypes.byref(cfg))


def _ptr(t: Optional[torch.Tensor]):
    return None if t is None else ctypes.c_void_p(t.data_ptr())


def _stream(stream) -> ctypes.c_void_p:
    if stream is None:
        stream = torch.cuda.current_stream()
    return ctypes.c_void_p(stream.cuda_stream)


def _need(t: torch.Tensor, dtype, name: str) -> None:
    if not t.is_cuda or t.dtype != dtype or not t.is_contiguous():
        raise ValueError(f"{name}: expected a contiguous CUDA {dtype} tensor, got "
                         f"{t.dtype} on {t.device} (contiguous={t.is_contiguous()})")


class MlaDecode:
    """One handle of the library: its configuration plus its device workspace."""

    def __init__(self, n_heads: int, max_batch: int, max_kv_len: int, page_size: int = 0,
                 softmax_scale: float = 0.0, rope_base: float = 10000.0, max_splits: int = 0,
                 device: Optional[int] = None, q_len: int = 1, **yarn):
        """`yarn`: yarn_factor, yarn_original_len, yarn_alpha, yarn_beta, yarn_mscale_coef
        (make_config). With q_len > 1 the per-sequence tensors carry a token axis:
        q_c [B, q_len, n_h, 128], q_abs [B, q_len, n_h, 576], latent [B, q_len, n_h, 512], ..."""
        self._lib = load_library()
        self.q_len = max(1, int(q_len))
        self.cfg = make_config(n_heads, max_batch, max_kv_len, page_size, softmax_scale,
                               rope_base, max_splits, q_len=q_len, **yarn)
        self.device = torch.cuda.current_device() if device is None else int(device)
        h = ctypes.c_void_p()
        _check(self._lib.mla_decode_create(ctypes.byref(self.cfg), self.device, ctypes.byref(h)),
               "mla_decode_create")
        self._h = h

    # -- lifetime ----------------------------------------------------------------------
    def close(self) -> None:
        if getattr(self, "_h", None) is not None and self._h.value is not None:
            _check(self._lib.mla_destroy(self._h), "mla_destroy")
            self._h = None

    def __del__(self):
        try:
            self.close()
        except Exception:
            pass

    def __enter__(self):
        return self

    def __exit__(self, *exc):
        self.close()

    @property
    def workspace_bytes(self) -> int:
        return int(self._lib.mla_workspace_bytes(self._h))

    # -- the three steps ---------------------------------------------------------------
    def absorb_q(self, q_c: torch.Tensor, q_r: torch.Tensor, w_uk: torch.Tensor,
                 kv_lens: torch.Tensor, q_abs: Optional[torch.Tensor] = None,
                 stream=None) -> torch.Tensor:
        B = q_c.shape[0]
        for t, n in ((q_c, "q_c"), (q_r, "q_r"), (w_uk, "w_uk")):
            _need(t, torch.bfloat16, n)
        _need(kv_lens, torch.int32, "kv_lens")
        if q_abs is None:
            q_abs = torch.empty(tuple(q_c.shape[:-1]) + (ROW,), dtype=torch.bfloat16, device=q_c.device)
        _need(q_abs, torch.bfloat16, "q_abs")
        _check(self._lib.mla_absorb_q(self._h, B, _ptr(q_c), _ptr(q_r), _ptr(w_uk), _ptr(kv_lens),
                                      _ptr(q_abs), _stream(stream)), "mla_absorb_q")
        return q_abs

    def append_kv(self, hidden: torch.Tensor, w_dkv: torch.Tensor, w_kr: torch.Tensor,
                  gamma: torch.Tensor, cache: torch.Tensor, kv_lens: torch.Tensor,
                  page_table: Optional[torch.Tensor] = None, eps: float = 1e-6,
                  stream=None) -> torch.Tensor:
        """Write the new token's cache row [RMSNorm(W_DKV h)*gamma ; RoPE(W_KR h)] as token
        kv_lens[b]-1 of every sequence b. hidden [B, d] bf16; w_dkv [512, d]; w_kr [64, d];
        gamma [512]; cache as for decode_attn. Returns the cache."""
        B, d = hidden.shape[0], hidden.shape[-1]
        for t, n in ((hidden, "hidden"), (w_dkv, "w_dkv"), (w_kr, "w_kr"), (gamma, "gamma")):
            _need(t, torch.bfloat16, n)
        _need(kv_lens, torch.int32, "kv_lens")
        row_stride, seq_stride, c_kv, k_r, max_pages, num_pages = self._cache_view(cache, page_table)
        _check(self._lib.mla_append_kv(
            self._h, B, d, _ptr(hidden), _ptr(w_dkv), _ptr(w_kr), _ptr(gamma), float(eps),
            ctypes.c_void_p(c_kv), ctypes.c_void_p(k_r), row_stride, seq_stride, _ptr(kv_lens),
            _ptr(page_table), max_pages, num_pages, _stream(stream)), "mla_append_kv")
        return cache

    def append_kv_fp8(self, hidden: torch.Tensor, w_dkv: torch.Tensor, w_kr: torch.Tensor,
                      gamma: torch.Tensor, codes: torch.Tensor, exps: torch.Tensor,
                      kv_lens: torch.Tensor, page_table: Optional[torch.Tensor] = None,
                      eps: float = 1e-6, stream=None):
        """append_kv into a quantised cache: codes uint8 [B, Lmax, 576] or [P, 64, 576], exps
        int8 shaped like codes[..., 0] (the layout of decode_attn_fp8)."""
        B, d = hidden.shape[0], hidden.shape[-1]
        for t, n in ((hidden, "hidden"), (w_dkv, "w_dkv"), (w_kr, "w_kr"), (gamma, "gamma")):
            _need(t, torch.bfloat16, n)
        _need(kv_lens, torch.int32, "kv_lens")
        if not codes.is_cuda or codes.dtype != torch.uint8 or codes.dim() != 3 or codes.stride(-1) != 1:
            raise ValueError("codes: expected a CUDA uint8 [*, *, 576] tensor with unit inner stride")
        _need(exps, torch.int8, "exps")
        row_stride = codes.stride(1)
        seq_stride = codes.stride(0) // row_stride
        if exps.shape != codes.shape[:2] or exps.stride(0) != seq_stride:
            raise ValueError("exps must index rows as codes does")
        max_pages = num_pages = 0
        if page_table is not None:
            _need(page_table, torch.int32, "page_table")
            max_pages, num_pages, seq_stride = page_table.shape[1], codes.shape[0], 0
        _check(self._lib.mla_append_kv_fp8(
            self._h, B, d, _ptr(hidden), _ptr(w_dkv), _ptr(w_kr), _ptr(gamma), float(eps),
            _ptr(codes), _ptr(exps), row_stride, seq_stride, _ptr(kv_lens), _ptr(page_table),
            max_pages, num_pages, _stream(stream)), "mla_append_kv_fp8")
        return codes, exps

    @staticmethod
    def _cache_view(cache: torch.Tensor, page_table: Optional[torch.Tensor]):
        if not cache.is_cuda or cache.dtype != torch.bfloat16 or cache.dim() != 3 or cache.stride(-1) != 1:
            raise ValueError("cache: expected a CUDA bf16 [*, *, 576] tensor with unit inner stride")
        row_stride = cache.stride(1)
        seq_stride = cache.stride(0) // row_stride
        c_kv = cache.data_ptr()
        k_r = c_kv + D_LATENT * cache.element_size()
        max_pages = num_pages = 0
        if page_table is not None:
            _need(page_table, torch.int32, "page_table")
            max_pages = page_table.shape[1]
            num_pages = cache.shape[0]
            seq_stride = 0
        return row_stride, seq_stride, c_kv, k_r, max_pages, num_pages

    def decode_attn(self, q_abs: torch.Tensor, cache: torch.Tensor, kv_lens: torch.Tensor,
                    page_table: Optional[torch.Tensor] = None,
                    out_latent: Optional[torch.Tensor] = None, lse: Optional[torch.Tensor] = None,
                    want_lse: bool = True, stream=None) -> Tuple[torch.Tensor, Optional[torch.Tensor]]:
        """cache: contiguous [B, Lmax, 576] or paged [num_pages, page_size, 576] bf16 rows
        [c^KV ; k^R]. Returns (out_latent [B, n_h, 512] bf16, lse [B, n_h] fp32 or None)."""
        B = q_abs.shape[0]
        _need(q_abs, torch.bfloat16, "q_abs")
        _need(kv_lens, torch.int32, "kv_lens")
        row_stride, seq_stride, c_kv, k_r, max_pages, num_pages = self._cache_view(cache, page_table)
        if out_latent is None:
            out_latent = torch.empty(tuple(q_abs.shape[:-1]) + (D_LATENT,), dtype=torch.bfloat16,
                                     device=q_abs.device)
        if lse is None and want_lse:
            lse = torch.empty(tuple(q_abs.shape[:-1]), dtype=torch.float32, device=q_abs.device)
        _check(self._lib.mla_decode_attn(
            self._h, B, _ptr(q_abs), ctypes.c_void_p(c_kv), ctypes.c_void_p(k_r), row_stride,
            seq_stride, _ptr(kv_lens), _ptr(page_table), max_pages, num_pages, _ptr(out_latent),
            _ptr(lse), _stream(stream)), "mla_decode_attn")
        return out_latent, lse

    def prefill_attn(self, q_abs: torch.Tensor, cache: torch.Tensor, kv_lens: torch.Tensor,
                     page_table: Optional[torch.Tensor] = None,
                     out_latent: Optional[torch.Tensor] = None, lse: Optional[torch.Tensor] = None,
                     want_lse: bool = True, stream=None) -> Tuple[torch.Tensor, Optional[torch.Tensor]]:
        """Prefill: the handle's q_len new tokens of every sequence, q_abs [B, T, n_h, 576], over
        the cache (as decode_attn), in one kernel. Returns (out_latent [B, T, n_h, 512] bf16,
        lse [B, T, n_h] fp32 or None); the same results as decode_attn with this handle."""
        B = q_abs.shape[0]
        _need(q_abs, torch.bfloat16, "q_abs")
        _need(kv_lens, torch.int32, "kv_lens")
        row_stride, seq_stride, c_kv, k_r, max_pages, num_pages = self._cache_view(cache, page_table)
        if out_latent is None:
            out_latent = torch.empty(tuple(q_abs.shape[:-1]) + (D_LATENT,), dtype=torch.bfloat16,
                                     device=q_abs.device)
        if lse is None and want_lse:
            lse = torch.empty(tuple(q_abs.shape[:-1]), dtype=torch.float32, device=q_abs.device)
        _check(self._lib.mla_prefill_attn(
            self._h, B, _ptr(q_abs), ctypes.c_void_p(c_kv), ctypes.c_void_p(k_r), row_stride,
            seq_stride, _ptr(kv_lens), _ptr(page_table), max_pages, num_pages, _ptr(out_latent),
            _ptr(lse), _stream(stream)), "mla_prefill_attn")
        return out_latent, lse

    def decode_attn_fp8(self, q_abs: torch.Tensor, codes: torch.Tensor, exps: torch.Tensor,
                        kv_lens: torch.Tensor, page_table: Optional[torch.Tensor] = None,
                        out_latent: Optional[torch.Tensor] = None, lse: Optional[torch.Tensor] = None,
                        want_lse: bool = True, stream=None):
        """Attention over a quantised cache: codes uint8 [B, Lmax, 576] or [P, 64, 576] (E4M3),
        exps int8 [B, Lmax] or [P, 64] (row r is 2^exps[r] times its codes' values)."""
        B = q_abs.shape[0]
        _need(q_abs, torch.bfloat16, "q_abs")
        _need(kv_lens, torch.int32, "kv_lens")
        if not codes.is_cuda or codes.dtype != torch.uint8 or codes.dim() != 3 or codes.stride(-1) != 1:
            raise ValueError("codes: expected a CUDA uint8 [*, *, 576] tensor with unit inner stride")
        _need(exps, torch.int8, "exps")
        if exps.stride(-1) != 1 or exps.shape != codes.shape[:2]:
            raise ValueError("exps: one int8 per cached row, shaped like codes[..., 0]")
        row_stride = codes.stride(1)
        seq_stride = codes.stride(0) // row_stride
        if exps.stride(0) != seq_stride:
            raise ValueError("exps must index rows as codes does")
        max_pages = num_pages = 0
        if page_table is not None:
            _need(page_table, torch.int32, "page_table")
            max_pages, num_pages, seq_stride = page_table.shape[1], codes.shape[0], 0
        if out_latent is None:
            out_latent = torch.empty(tuple(q_abs.shape[:-1]) + (D_LATENT,), dtype=torch.bfloat16,
                                     device=q_abs.device)
        if lse is None and want_lse:
            lse = torch.empty(tuple(q_abs.shape[:-1]), dtype=torch.float32, device=q_abs.device)
        _check(self._lib.mla_decode_attn_fp8(
            self._h, B, _ptr(q_abs), _ptr(codes), _ptr(exps), row_stride, seq_stride, _ptr(kv_lens),
            _ptr(page_table), max_pages, num_pages, _ptr(out_latent), _ptr(lse), _stream(stream)),
            "mla_decode_attn_fp8")
        return out_latent, lse

    def decode_attn_partial(self, q_abs: torch.Tensor, cache: torch.Tensor, kv_lens: torch.Tensor,
                            page_table: Optional[torch.Tensor] = None,
                            out_latent: Optional[torch.Tensor] = None,
                            lse: Optional[torch.Tensor] = None,
                            stream=None) -> Tuple[torch.Tensor, torch.Tensor]:
        """Attention over the cache rows this caller holds (one shard of each sequence):
        (latent fp32 [B, (T,) n_h, 512], lse fp32 [B, (T,) n_h]), to be merged across shards
        with merge_partials. q_abs is rotated at the request's global positions."""
        B = q_abs.shape[0]
        _need(q_abs, torch.bfloat16, "q_abs")
        _need(kv_lens, torch.int32, "kv_lens")
        row_stride, seq_stride, c_kv, k_r, max_pages, num_pages = self._cache_view(cache, page_table)
        if out_latent is None:
            out_latent = torch.empty(tuple(q_abs.shape[:-1]) + (D_LATENT,), dtype=torch.float32,
                                     device=q_abs.device)
        if lse is None:
            lse = torch.empty(tuple(q_abs.shape[:-1]), dtype=torch.float32, device=q_abs.device)
        _need(out_latent, torch.float32, "out_latent")
        _need(lse, torch.float32, "lse")
        _check(self._lib.mla_decode_attn_partial(
            self._h, B, _ptr(q_abs), ctypes.c_void_p(c_kv), ctypes.c_void_p(k_r), row_stride,
            seq_stride, _ptr(kv_lens), _ptr(page_table), max_pages, num_pages, _ptr(out_latent),
            _ptr(lse), _stream(stream)), "mla_decode_attn_partial")
        return out_latent, lse

    def merge_partials(self, latent_parts: torch.Tensor, lse_parts: torch.Tensor,
                       out_latent: Optional[torch.Tensor] = None,
                       lse: Optional[torch.Tensor] = None, want_lse: bool = True,
                       stream=None) -> Tuple[torch.Tensor, Optional[torch.Tensor]]:
        """latent_parts fp32 [P, B, (T,) n_h, 512], lse_parts fp32 [P, B, (T,) n_h] ->
        (latent bf16 [B, (T,) n_h, 512], lse fp32 or None)."""
        _need(latent_parts, torch.float32, "latent_parts")
        _need(lse_parts, torch.float32, "lse_parts")
        P, B = latent_parts.shape[0], latent_parts.shape[1]
        if out_latent is None:
            out_latent = torch.empty(tuple(latent_parts.shape[1:]), dtype=torch.bfloat16,
                                     device=latent_parts.device)
        if lse is None and want_lse:
            lse = torch.empty(tuple(lse_parts.shape[1:]), dtype=torch.float32, device=lse_parts.device)
        _check(self._lib.mla_merge_partials(self._h, B, P, _ptr(latent_parts), _ptr(lse_parts),
                                            _ptr(out_latent), _ptr(lse), _stream(stream)),
               "mla_merge_partials")
        return out_latent, lse

    def apply_wuv(self, latent: torch.Tensor, w_uv: torch.Tensor,
                  out: Optional[torch.Tensor] = None, stream=None) -> torch.Tensor:
        B = latent.shape[0]
        _need(latent, torch.bfloat16, "latent")
        _need(w_uv, torch.bfloat16, "w_uv")
        if out is None:
            out = torch.empty(tuple(latent.shape[:-1]) + (128,), dtype=torch.bfloat16, device=latent.device)
        _need(out, torch.bfloat16, "out")
        _check(self._lib.mla_apply_wuv(self._h, B, _ptr(latent), _ptr(w_uv), _ptr(out),
                                       _stream(stream)), "mla_apply_wuv")
        return out

    @staticmethod
    def _fp8_weight(codes: torch.Tensor, exps: torch.Tensor, n_heads: int, what: str):
        if not codes.is_cuda or codes.dtype != torch.uint8 or not codes.is_contiguous() or \
                codes.numel() != n_heads * 128 * D_LATENT:
            raise ValueError(f"{what} codes: expected a contiguous CUDA uint8 [n_h * 128, 512] tensor")
        if not exps.is_cuda or exps.dtype != torch.int8 or not exps.is_contiguous() or \
                exps.numel() != n_heads * 128 * (D_LATENT // 128):
            raise ValueError(f"{what} exponents: expected a contiguous CUDA int8 [n_h * 128, 4] tensor")

    def absorb_q_fp8(self, q_c: torch.Tensor, q_r: torch.Tensor, w_uk_codes: torch.Tensor,
                     w_uk_exp: torch.Tensor, kv_lens: torch.Tensor,
                     q_abs: Optional[torch.Tensor] = None, stream=None) -> torch.Tensor:
        """absorb_q with W_UK as E4M3 codes [n_h * 128, 512] and one int8 exponent per 1 x 128
        tile [n_h * 128, 4] (W = value(code) * 2^exp)."""
        B = q_c.shape[0]
        for t, n in ((q_c, "q_c"), (q_r, "q_r")):
            _need(t, torch.bfloat16, n)
        _need(kv_lens, torch.int32, "kv_lens")
        self._fp8_weight(w_uk_codes, w_uk_exp, self.cfg.n_heads, "w_uk")
        if q_abs is None:
            q_abs = torch.empty(tuple(q_c.shape[:-1]) + (ROW,), dtype=torch.bfloat16, device=q_c.device)
        _need(q_abs, torch.bfloat16, "q_abs")
        _check(self._lib.mla_absorb_q_fp8(self._h, B, _ptr(q_c), _ptr(q_r), _ptr(w_uk_codes),
                                          _ptr(w_uk_exp), _ptr(kv_lens), _ptr(q_abs), _stream(stream)),
               "mla_absorb_q_fp8")
        return q_abs

    def apply_wuv_fp8(self, latent: torch.Tensor, w_uv_codes: torch.Tensor, w_uv_exp: torch.Tensor,
                      out: Optional[torch.Tensor] = None, stream=None) -> torch.Tensor:
        """apply_wuv with W_UV as E4M3 codes and per-tile exponents (as absorb_q_fp8)."""
        B = latent.shape[0]
        _need(latent, torch.bfloat16, "latent")
        self._fp8_weight(w_uv_codes, w_uv_exp, self.cfg.n_heads, "w_uv")
        if out is None:
            out = torch.empty(tuple(latent.shape[:-1]) + (128,), dtype=torch.bfloat16, device=latent.device)
        _need(out, torch.bfloat16, "out")
        _check(self._lib.mla_apply_wuv_fp8(self._h, B, _ptr(latent), _ptr(w_uv_codes), _ptr(w_uv_exp),
                                           _ptr(out), _stream(stream)), "mla_apply_wuv_fp8")
        return out

    def step(self, q_c, q_r, w_uk, w_uv, cache, kv_lens, page_table=None, stream=None,
             bufs: Optional[dict] = None):
        """One decode step in one C call (mla_decode_step): absorb -> split-KV attention -> W_UV,
        the same results as the three calls, with the work plan built beside the absorption.
        Returns the head outputs [B, (T,) n_h, 128] bf16. `bufs` may hold preallocated q_abs /
        latent / out; q_abs and latent are left holding the intermediate results."""
        bufs = bufs or {}
        B = q_c.shape[0]
        for t, n in ((q_c, "q_c"), (q_r, "q_r"), (w_uk, "w_uk"), (w_uv, "w_uv")):
            _need(t, torch.bfloat16, n)
        _need(kv_lens, torch.int32, "kv_lens")
        row_stride, seq_stride, c_kv, k_r, max_pages, num_pages = self._cache_view(cache, page_table)
        lead = tuple(q_c.shape[:-1])
        q_abs, latent, out = bufs.get("q_abs"), bufs.get("latent"), bufs.get("out")
        if q_abs is None:
            q_abs = torch.empty(lead + (ROW,), dtype=torch.bfloat16, device=q_c.device)
        if latent is None:
            latent = torch.empty(lead + (D_LATENT,), dtype=torch.bfloat16, device=q_c.device)
        if out is None:
            out = torch.empty(lead + (128,), dtype=torch.bfloat16, device=q_c.device)
        for t, n in ((q_abs, "q_abs"), (latent, "latent"), (out, "out")):
            _need(t, torch.bfloat16, n)
        _check(self._lib.mla_decode_step(
            self._h, B, _ptr(q_c), _ptr(q_r), _ptr(w_uk), _ptr(w_uv), ctypes.c_void_p(c_kv),
            ctypes.c_void_p(k_r), row_stride, seq_stride, _ptr(kv_lens), _ptr(page_table), max_pages,
            num_pages, _ptr(q_abs), _ptr(latent), _ptr(out), _stream(stream)), "mla_decode_step")
        return out

    def check_device_errors(self, stream=None) -> int:
        """Synchronise the stream; raise MlaError if a kernel set the device error word."""
        word = ctypes.c_uint32(0)
        st = self._lib.mla_check_device_errors(self._h, _stream(stream), ctypes.byref(word))
        if st != MLA_OK:
            raise MlaError(st, "device check", int(word.value))
        return 0
