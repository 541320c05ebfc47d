"""Sequence split across GPUs, for contexts longer than one GPU should hold.

A sequence's cached pages are cut into contiguous page ranges ("shards");
shard r lives in GPU r's cache.  Each GPU decodes every query row over its
own shard (``mla_decode_packed`` with one query per row and the row's
visible rows inside the shard as its length), takes per-row ``(o_lat, lse)``
with ``mla_combine_lse``, the pairs of all GPUs are all-gathered (NCCL over
NVLink; a few hundred KiB per query row), and ``mla_merge_shards`` merges
them into the decode over the whole sequence.

The pages motivate long contexts ("Multi-head Latent Attention (MLA) Nedir?",
section "Sayılarla MLA": reasoning chains of tens of thousands of tokens);
the merge is the split combine's log-sum-exp merge one level up, which the
pages do not describe.  This module only plans and marshals: the decode,
the per-shard combine and the merge are the library's kernels.
"""

from __future__ import annotations

import contextlib
from dataclasses import dataclass
from typing import List, Optional, Sequence, Tuple

import torch

from . import abi


@dataclass
class ShardPlan:
    """How ``n_shards`` GPUs split the keys of ``batch * n_q`` query rows.

    ``page_bounds[b, r]`` .. ``page_bounds[b, r + 1]`` are the pages of
    sequence ``b`` in shard ``r`` (contiguous, about equal counts).  For shard
    ``r``, ``block_tables[r][v]`` lists the block ids of those pages for query
    row ``v = b * n_q + j`` (unused entries 0) and ``seq_lens[r][v]`` the rows
    of them that query ``j`` sees (0 when none)."""

    n_shards: int
    n_q: int
    block_size: int
    page_bounds: torch.Tensor           # int64 [batch, n_shards + 1]
    block_tables: List[torch.Tensor]    # per shard int32 [batch * n_q, max pages of a shard]
    seq_lens: List[torch.Tensor]        # per shard int32 [batch * n_q]


def shard_plan(block_table: torch.Tensor, seq_lens: torch.Tensor, n_q: int, block_size: int,
               n_shards: int) -> ShardPlan:
    """Cut every sequence's pages into ``n_shards`` contiguous ranges (host
    work on CPU tensors).  ``seq_lens`` counts each sequence's rows including
    its ``n_q`` new ones, as for ``mla_decode``; query ``j`` of sequence
    ``b`` sees rows ``0 .. seq_lens[b] - n_q + j``."""
    if n_shards < 1 or n_q < 1 or block_size < 1:
        raise ValueError("n_shards, n_q and block_size must be positive")
    bt = block_table.to("cpu", torch.int64)
    lens = seq_lens.to("cpu", torch.int64)
    batch = lens.numel()
    if bt.dim() != 2 or bt.shape[0] != batch:
        raise ValueError("block_table must be [batch, max_blocks]")
    if bool((lens < n_q).any()) or bool((lens > bt.shape[1] * block_size).any()):
        raise ValueError("every sequence needs n_q <= seq_lens[b] <= max_blocks * block_size")
    pages = (lens + block_size - 1) // block_size
    r = torch.arange(n_shards + 1, dtype=torch.int64)
    bounds = (pages[:, None] * r[None, :]) // n_shards          # [batch, n_shards + 1]
    width = max(1, int((bounds[:, 1:] - bounds[:, :-1]).max()))
    rows = batch * n_q
    b_of = torch.arange(rows) // n_q
    vis = lens[b_of] - n_q + torch.arange(rows) % n_q + 1        # rows each query sees
    tables, lengths = [], []
    col = torch.arange(width, dtype=torch.int64)
    for s in range(n_shards):
        lo, hi = bounds[b_of, s], bounds[b_of, s + 1]
        idx = lo[:, None] + col[None, :]
        inside = idx < hi[:, None]
        t = torch.where(inside, bt[b_of[:, None], idx.clamp(max=bt.shape[1] - 1)], torch.zeros_like(idx))
        tables.append(t.to(torch.int32).contiguous())
        n = (vis - lo * block_size).clamp(min=0)
        lengths.append(torch.minimum(n, (hi - lo) * block_size).to(torch.int32).contiguous())
    return ShardPlan(n_shards, n_q, block_size, bounds, tables, lengths)


def gather_partials(o_lat: torch.Tensor, lse: torch.Tensor, group=None) -> Tuple[torch.Tensor, torch.Tensor]:
    """All ranks' ``(o_lat, lse)`` stacked in rank order: ``[world, ...]``.
    Without an initialised process group (one GPU) the local pair alone."""
    import torch.distributed as dist
    if not (dist.is_available() and dist.is_initialized()):
        return o_lat.unsqueeze(0), lse.unsqueeze(0)
    world = dist.get_world_size(group)
    o_parts = torch.empty((world,) + tuple(o_lat.shape), dtype=o_lat.dtype, device=o_lat.device)
    lse_parts = torch.empty((world,) + tuple(lse.shape), dtype=lse.dtype, device=lse.device)
    if dist.get_backend(group) == "nccl":   # one flat gather each, straight into the stacked buffers
        dist.all_gather_into_tensor(o_parts, o_lat.contiguous(), group=group)
        dist.all_gather_into_tensor(lse_parts, lse.contiguous(), group=group)
    else:
        dist.all_gather(list(o_parts.unbind(0)), o_lat.contiguous(), group=group)
        dist.all_gather(list(lse_parts.unbind(0)), lse.contiguous(), group=group)
    return o_parts, lse_parts


def decode_shard(cfg: abi.Config, q_packed: torch.Tensor, rows: int, cache: abi.Cache, seq_lens: torch.Tensor,
                 workspace: torch.Tensor, o_lat: torch.Tensor, lse: torch.Tensor, max_workers: int = 0,
                 stream=None) -> None:
    """This GPU's shard: every query row over the shard's rows (one query per
    row), then its ``(o_lat, lse)``.  The decode is the packed (tensor-core)
    one: for an FP8 cache, expand the shard's pages first
    (``mla_cache_dequant_fp8``) and pass the scratch cache with the
    configuration without ``fp8_cache``."""
    abi.mla_decode_packed(cfg, q_packed, rows, 1, cache, seq_lens, workspace, max_workers, stream)
    abi.mla_combine_lse(cfg, workspace, rows, 1, o_lat, lse, stream)


def decode_sharded(cfg: abi.Config, q_packed: torch.Tensor, rows: int, caches: Sequence[abi.Cache],
                   seq_lens: Sequence[torch.Tensor], workspace: torch.Tensor, o_lat: torch.Tensor,
                   lse: Optional[torch.Tensor] = None, group=None, max_workers: int = 0,
                   stream=None) -> None:
    """The decode of ``rows`` query rows split over shards.

    With a process group of ``world`` ranks, ``caches`` / ``seq_lens`` hold
    this rank's shard only: it is decoded here, the pairs are all-gathered
    and merged on every rank.  Without one, all shards are given and decoded
    one after the other on this GPU (the same arithmetic, the exchange being
    a stack), e.g. to check the split against the unsplit decode."""
    H, d_c = cfg.n_heads, cfg.d_c
    dev = q_packed.device
    local = len(caches)
    o_loc = torch.empty(local, rows, H, d_c, dtype=torch.float32, device=dev)
    lse_loc = torch.empty(local, rows, H, dtype=torch.float32, device=dev)
    for r in range(local):
        decode_shard(cfg, q_packed, rows, caches[r], seq_lens[r], workspace, o_loc[r], lse_loc[r], max_workers,
                     stream)
    import torch.distributed as dist
    if dist.is_available() and dist.is_initialized():
        if local != 1:
            raise ValueError("with a process group each rank decodes exactly its own shard")
        with torch.cuda.stream(stream) if stream is not None else contextlib.nullcontext():
            o_parts, lse_parts = gather_partials(o_loc[0], lse_loc[0], group)
    else:
        o_parts, lse_parts = o_loc, lse_loc
    abi.mla_merge_shards(cfg, o_parts, lse_parts, o_lat, lse, stream)

