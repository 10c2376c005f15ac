"""A long request whose cached tokens are spread over several GPUs, one process per GPU.

Each rank holds one contiguous range of every sequence's tokens (whole 64-token tiles, so a
paged cache holds whole pages). A decode step then runs, on every rank:
  1. mla_absorb_q with the GLOBAL kv_lens (the query sits at the request's last position; the
     cached k^R rows were rotated at their global positions when they were written);
  2. mla_decode_attn_partial over the rows this rank holds -> (latent fp32, lse);
  3. an all-gather of (latent, lse) over the process group (NCCL over NVLink on GPUs);
  4. mla_merge_partials -> the latent of the whole request (the log-sum-exp merge), then
     mla_apply_wuv.
The exchange is one all-gather of B x rows x 513 floats per rank (about 262 KB for one
128-head sequence); the merge runs in the library's kernel. A rank that holds no rows of a
sequence contributes lse = -inf, which the merge ignores.
"""

from __future__ import annotations

from typing import List, Optional, Sequence, Tuple

import torch
import torch.distributed as dist

TILE = 64


def shard_ranges(kv_len: int, world: int, tile: int = TILE) -> List[Tuple[int, int]]:
    """Token ranges [start, end) per rank: contiguous, in rank order, cut on tile boundaries,
    the tiles dealt as evenly as they allow (the first kv_len_tiles % world ranks get one
    more). Ranks past the last tile get empty ranges."""
    if kv_len < 0 or world < 1:
        raise ValueError("kv_len >= 0 and world >= 1")
    tiles = (kv_len + tile - 1) // tile
    per, extra = divmod(tiles, world)
    out, t0 = [], 0
    for r in range(world):
        n = per + (1 if r < extra else 0)
        start, end = min(kv_len, t0 * tile), min(kv_len, (t0 + n) * tile)
        out.append((start, end))
        t0 += n
    return out


def local_lengths(kv_lens: Sequence[int], rank: int, world: int) -> List[int]:
    """Rows of each sequence that `rank` holds."""
    out = []
    for L in kv_lens:
        start, end = shard_ranges(int(L), world)[rank]
        out.append(end - start)
    return out


def gather_partials(latent: torch.Tensor, lse: torch.Tensor, group=None) -> Tuple[torch.Tensor, torch.Tensor]:
    """All-gather every rank's (latent, lse) into [world, ...] tensors in rank order."""
    world = dist.get_world_size(group)
    out = []
    for t in (latent, lse):
        flat = torch.empty(world * t.numel(), dtype=t.dtype, device=t.device)   # rank-major
        dist.all_gather_into_tensor(flat, t.contiguous().view(-1), group=group)
        out.append(flat.view((world,) + tuple(t.shape)))
    return out[0], out[1]


class ShardedDecode:
    """The decode step of a request whose KV rows are sharded across the process group.
    `handle` is this rank's binding.MlaDecode (max_kv_len sized for the local rows)."""

    def __init__(self, handle, group=None):
        self.h = handle
        self.group = group

    def attention(self, q_abs: torch.Tensor, local_cache: torch.Tensor, local_kv_lens: torch.Tensor,
                  page_table: Optional[torch.Tensor] = None, want_lse: bool = True):
        latent, lse = self.h.decode_attn_partial(q_abs, local_cache, local_kv_lens, page_table)
        lat_all, lse_all = gather_partials(latent, lse, self.group)
        return self.h.merge_partials(lat_all, lse_all, want_lse=want_lse)

    def step(self, q_c, q_r, w_uk, w_uv, global_kv_lens, local_cache, local_kv_lens, page_table=None):
        q_abs = self.h.absorb_q(q_c, q_r, w_uk, global_kv_lens)
        latent, _ = self.attention(q_abs, local_cache, local_kv_lens, page_table, want_lse=False)
        return self.h.apply_wuv(latent, w_uv)
