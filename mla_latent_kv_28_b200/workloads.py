"""Seeded synthetic inputs for the MLA decode step.

This module is shared by the tests, the benchmark and the oracle checks. It holds only
random draws, their distributions and the memory layout of the inputs: none of the
method's arithmetic (no projection, rotation, softmax or sum of the decode step).

Recipe (every draw comes from one torch CPU generator seeded with `seed`, in this order:
weights, q^C, q^R, kv lengths, cache, page assignment):
  * W_UK, W_UV [n_h, d_h, d_c]: N(0, std = 1/sqrt(d_c)) in fp32, rounded to bf16 (RNE);
    fan-in is d_c because both map a latent c (d_c) to a head vector (d_h).
  * q^C [B, n_h, d_h], q^R [B, n_h, d_R]: N(0, 1) rounded to bf16. q^R is un-rotated;
    the decode step rotates it.
  * cache rows [c^KV (d_c) ; k^R (d_R)]: N(0, 1) rounded to bf16. k^R is the cached key,
    already rotated when it was written; a rotation of i.i.d. N(0,1) pairs is again
    i.i.d. N(0,1), so the draw has the distribution of a rotated key.
    With latent_scale="lognormal" each token's c^KV is multiplied by s_j ~ LogNormal(0, 0.5)
    before rounding (k^R is not scaled).
  * kv lengths: an int (all equal), a list, or ("uniform", lo, hi) drawn inclusive.
  * cache write of a new token (draw_append_inputs, its own generator): hidden h [B, d]
    N(0, 1); W_DKV [512, d] and W_KR [64, d] N(0, std = 1/sqrt(d)) (fan-in d); the latent
    RMSNorm weight gamma [512] = 1 + 0.1 N(0, 1); all rounded to bf16. d = 5120 is
    DeepSeek-V2's hidden size.
  * contiguous layout: cache [B, Lmax, 576]; rows at or past kv_len[b] are NaN.
  * paged layout: ceil(L_b / page_size) pages per sequence plus `spare_pages` spares form
    the physical pool [P, page_size, 576]; a seeded random permutation places the pages;
    page_table [B, ceil(Lmax / page_size)] int32 with -1 in unused entries; page tails
    past kv_len and the spare pages are NaN, so any read of a row that is not part of a
    sequence shows up as NaN in the output.
"""

from __future__ import annotations

import math
from dataclasses import dataclass
from typing import Optional, Sequence, Union

import torch

D_HEAD = 128
D_LATENT = 512
D_ROPE = 64
ROW = D_LATENT + D_ROPE

KvLenSpec = Union[int, Sequence[int], tuple]


@dataclass
class Workload:
    name: str
    batch: int
    n_heads: int
    kv_lens: torch.Tensor                 # int32 [B]
    q_c: torch.Tensor                     # bf16 [B, n_h, d_h]
    q_r: torch.Tensor                     # bf16 [B, n_h, d_R]
    w_uk: torch.Tensor                    # bf16 [n_h, d_h, d_c]
    w_uv: torch.Tensor                    # bf16 [n_h, d_h, d_c]
    cache: torch.Tensor                   # bf16 [B, Lmax, 576] or [P, page_size, 576]
    page_table: Optional[torch.Tensor]    # int32 [B, max_pages] or None
    page_size: int
    rope_base: float
    max_kv_len: int

    @property
    def cached_tokens(self) -> int:
        return int(self.kv_lens.to(torch.int64).sum())

    @property
    def num_pages(self) -> int:
        return int(self.cache.shape[0]) if self.page_size else 0

    def to(self, device) -> "Workload":
        def mv(t):
            return None if t is None else t.to(device)
        return Workload(self.name, self.batch, self.n_heads, mv(self.kv_lens), mv(self.q_c),
                        mv(self.q_r), mv(self.w_uk), mv(self.w_uv), mv(self.cache),
                        mv(self.page_table), self.page_size, self.rope_base, self.max_kv_len)


def _draw_lengths(spec: KvLenSpec, batch: int, gen: torch.Generator) -> torch.Tensor:
    if isinstance(spec, int):
        return torch.full((batch,), spec, dtype=torch.int32)
    if isinstance(spec, tuple) and len(spec) == 3 and spec[0] == "uniform":
        lo, hi = int(spec[1]), int(spec[2])
        return torch.randint(lo, hi + 1, (batch,), generator=gen, dtype=torch.int64).to(torch.int32)
    lens = torch.tensor(list(spec), dtype=torch.int32)
    assert lens.numel() == batch, "one kv length per sequence"
    return lens


def _randn_bf16(shape, gen, chunk_rows: int = 1 << 16) -> torch.Tensor:
    """N(0,1) rounded to bf16, drawn in row chunks to bound the fp32 temporary."""
    out = torch.empty(shape, dtype=torch.bfloat16)
    flat = out.view(-1, shape[-1])
    for r0 in range(0, flat.shape[0], chunk_rows):
        r1 = min(flat.shape[0], r0 + chunk_rows)
        flat[r0:r1] = torch.randn((r1 - r0, shape[-1]), generator=gen).to(torch.bfloat16)
    return out


def _draw_cache_rows(n_rows: int, latent_scale: str, gen: torch.Generator,
                     chunk_rows: int = 1 << 16) -> torch.Tensor:
    rows = torch.empty((n_rows, ROW), dtype=torch.bfloat16)
    for r0 in range(0, n_rows, chunk_rows):
        r1 = min(n_rows, r0 + chunk_rows)
        x = torch.randn((r1 - r0, ROW), generator=gen)
        if latent_scale == "lognormal":
            s = torch.exp(0.5 * torch.randn((r1 - r0, 1), generator=gen))
            x[:, :D_LATENT] *= s
        elif latent_scale != "none":
            raise ValueError(f"unknown latent_scale {latent_scale!r}")
        rows[r0:r1] = x.to(torch.bfloat16)
    return rows


def make_workload(batch: int, n_heads: int, kv_lens: KvLenSpec, *, page_size: int = 0,
                  rope_base: float = 10000.0, latent_scale: str = "none", seed: int = 0,
                  spare_pages: int = 16, max_kv_len: Optional[int] = None,
                  name: str = "custom") -> Workload:
    gen = torch.Generator().manual_seed(seed)
    wstd = 1.0 / math.sqrt(D_LATENT)
    w_uk = (torch.randn((n_heads, D_HEAD, D_LATENT), generator=gen) * wstd).to(torch.bfloat16)
    w_uv = (torch.randn((n_heads, D_HEAD, D_LATENT), generator=gen) * wstd).to(torch.bfloat16)
    q_c = _randn_bf16((batch, n_heads, D_HEAD), gen)
    q_r = _randn_bf16((batch, n_heads, D_ROPE), gen)
    lens = _draw_lengths(kv_lens, batch, gen)
    lmax = int(lens.max()) if batch > 0 else 0
    if max_kv_len is None:
        max_kv_len = lmax
    assert lmax <= max_kv_len

    nan = torch.tensor(float("nan"), dtype=torch.bfloat16)
    if page_size == 0:
        alloc = max(lmax, 1)
        cache = _draw_cache_rows(batch * alloc, latent_scale, gen).view(batch, alloc, ROW)
        for b in range(batch):
            cache[b, int(lens[b]):, :] = nan
        page_table = None
    else:
        pages_per_seq = [(int(L) + page_size - 1) // page_size for L in lens]
        n_pages = sum(pages_per_seq) + spare_pages
        cache = _draw_cache_rows(n_pages * page_size, latent_scale, gen).view(n_pages, page_size, ROW)
        perm = torch.randperm(n_pages, generator=gen).to(torch.int32)
        max_pages = max(1, (max_kv_len + page_size - 1) // page_size)
        page_table = torch.full((batch, max_pages), -1, dtype=torch.int32)
        used = torch.zeros(n_pages, dtype=torch.bool)
        off = 0
        for b in range(batch):
            n = pages_per_seq[b]
            page_table[b, :n] = perm[off:off + n]
            used[perm[off:off + n].long()] = True
            L = int(lens[b])
            if n and L % page_size:
                cache[int(perm[off + n - 1]), L % page_size:, :] = nan
            off += n
        cache[~used] = nan
    return Workload(name, batch, n_heads, lens, q_c, q_r, w_uk, w_uv, cache, page_table,
                    page_size, float(rope_base), int(max_kv_len))


# The five workloads of the decode step, named by what they are.
CONFIGS = {
    # batch 1, 16 heads, 256 cached tokens; RoPE off (the workload does not mention it)
    "tiny_h16_l256": dict(batch=1, n_heads=16, kv_lens=256, rope_base=0.0),
    # DeepSeek-V2-shaped layer: batch 32, 128 heads, 4096 cached tokens each
    "v2_b32_l4096": dict(batch=32, n_heads=128, kv_lens=4096, rope_base=10000.0),
    # long context: batch 4 x 32768 tokens
    "long_b4_l32768": dict(batch=4, n_heads=128, kv_lens=32768, rope_base=10000.0),
    # one 128K request, per-token LogNormal(0, 0.5) scale on the latents
    "single_l131072_lognormal": dict(batch=1, n_heads=128, kv_lens=131072, rope_base=10000.0,
                                     latent_scale="lognormal"),
    # ragged paged batch: 64 sequences, lengths U[1, 16384], 64-token pages
    "ragged_paged_b64": dict(batch=64, n_heads=128, kv_lens=("uniform", 1, 16384),
                             page_size=64, rope_base=10000.0, max_kv_len=16384),
}


def config_workload(name: str, seed: int = 0) -> Workload:
    kw = dict(CONFIGS[name])
    return make_workload(seed=seed, name=name, **kw)


def draw_q_abs(batch: int, n_heads: int, seed: int = 1) -> torch.Tensor:
    """A stand-alone absorbed-query input [B, n_h, 576] bf16 for testing the attention call
    by itself: the first 512 values N(0, 0.5^2) (the spread of W_UK^T q^C under the weight
    recipe above), the last 64 N(0, 1)."""
    gen = torch.Generator().manual_seed(seed)
    q = torch.randn((batch, n_heads, ROW), generator=gen)
    q[..., :D_LATENT] *= 0.5
    return q.to(torch.bfloat16)


def draw_latent(batch: int, n_heads: int, seed: int = 2) -> torch.Tensor:
    """A stand-alone latent input [B, n_h, 512] bf16 ~ N(0, 1) for testing the W_UV call."""
    gen = torch.Generator().manual_seed(seed)
    return torch.randn((batch, n_heads, D_LATENT), generator=gen).to(torch.bfloat16)


def draw_append_inputs(batch: int, d_model: int = 5120, seed: int = 3) -> dict:
    """Inputs of the cache write of one decode step: hidden [B, d], w_dkv [512, d],
    w_kr [64, d], gamma [512], all bf16 (recipe above)."""
    gen = torch.Generator().manual_seed(seed)
    wstd = 1.0 / math.sqrt(d_model)
    hidden = _randn_bf16((batch, d_model), gen)
    w_dkv = (torch.randn((D_LATENT, d_model), generator=gen) * wstd).to(torch.bfloat16)
    w_kr = (torch.randn((D_ROPE, d_model), generator=gen) * wstd).to(torch.bfloat16)
    gamma = (1.0 + 0.1 * torch.randn((D_LATENT,), generator=gen)).to(torch.bfloat16)
    return {"hidden": hidden, "w_dkv": w_dkv, "w_kr": w_kr, "gamma": gamma}


def draw_token_queries(batch: int, q_len: int, n_heads: int, seed: int = 4):
    """Queries of q_len new tokens per sequence: q^C [B, T, n_h, 128] and q^R [B, T, n_h, 64],
    N(0, 1) rounded to bf16 (the one-token recipe with a token axis)."""
    gen = torch.Generator().manual_seed(seed)
    q_c = _randn_bf16((batch, q_len, n_heads, D_HEAD), gen)
    q_r = _randn_bf16((batch, q_len, n_heads, D_ROPE), gen)
    return q_c, q_r
