"""Context parallelism for long requests: the keys of every request are split into contiguous,
page-aligned ranges, one per rank; each rank decodes its range with the ordinary decode (a page
table that lists only its pages), the ranks exchange (out, lse) with one all-gather over NCCL, and
every rank merges the parts with the library's LSE merge (mla_merge_lse_parts_bf16).

Why the ordinary decode serves a key range: with one query token per request (q_len 1) the query
sees every stored key, so a range of n keys is decoded as a request with cache length n - 1 whose
page table holds the range's pages.  Ranges start on page boundaries, so the slots inside a page
are unchanged.  A rank whose range of some request is empty decodes a one-key stand-in and reports
lse = -inf for it, which the merge skips.  q_len > 1 is not supported (the causal rule among the
step's new tokens would need per-query ranges).

Only argument marshalling and the exchange happen here; the decode and the merge are CUDA kernels.
"""
from __future__ import annotations

from dataclasses import dataclass

import numpy as np
import torch

from . import _lib


@dataclass
class LocalShard:
    """One rank's view of a batch: its page table, cache lengths and which requests it has no keys of."""
    lookup_table: torch.Tensor          # int32 view of uint32 [B, local_max_pages]
    scales_lookup_table: torch.Tensor | None
    cache_lengths: torch.Tensor         # int32 view of uint32 [B]: local keys - 1 (0 for empty ranges)
    empty: torch.Tensor                 # bool [B]: this rank holds none of request b's keys
    max_cache_length: int
    first_page: np.ndarray              # [B] first logical page of the range
    num_keys: np.ndarray                # [B] keys in the range


def page_ranges(cache_lengths, page_size: int, world: int, max_prompt_length: int = 1):
    """Per rank, the logical pages [first, first + count) of each request's n_b = L_b + T keys:
    ceil(pages_b / world) pages per rank, the last ranks getting fewer or none."""
    L = np.asarray(cache_lengths, dtype=np.int64)
    n = L + int(max_prompt_length)
    pages = (n + page_size - 1) // page_size
    per = (pages + world - 1) // world
    out = []
    for r in range(world):
        first = np.minimum(r * per, pages)
        count = np.minimum(pages, (r + 1) * per) - first
        keys = np.clip(n - first * page_size, 0, count * page_size)
        out.append((first, count, keys))
    return out


def local_shard(lookup_table, cache_lengths, page_size: int, world: int, rank: int,
                scales_lookup_table=None, device=None) -> LocalShard:
    """Rank `rank`'s page tables and lengths (host tables in, tensors on `device` out)."""
    lut = np.asarray(lookup_table).astype(np.int64) & 0xFFFFFFFF
    slut = None if scales_lookup_table is None else (np.asarray(scales_lookup_table).astype(np.int64) & 0xFFFFFFFF)
    first, count, keys = page_ranges(cache_lengths, page_size, world)[rank]
    B = lut.shape[0]
    width = max(1, int(count.max()) if B else 1)
    loc = np.zeros((B, width), dtype=np.int64)
    sloc = None if slut is None else np.zeros((B, width), dtype=np.int64)
    empty = keys == 0
    for b in range(B):
        if empty[b]:
            loc[b, 0] = lut[b, 0]                        # a valid page for the one-key stand-in
            if sloc is not None:
                sloc[b, 0] = slut[b, 0]
            continue
        loc[b, :count[b]] = lut[b, first[b]:first[b] + count[b]]
        if sloc is not None:
            sloc[b, :count[b]] = slut[b, first[b]:first[b] + count[b]]
    lens = np.where(empty, 0, keys - 1)

    def i32(a):
        return torch.from_numpy(a.astype(np.uint32).view(np.int32).copy()).to(device)

    return LocalShard(lookup_table=i32(loc), scales_lookup_table=None if sloc is None else i32(sloc),
                      cache_lengths=i32(lens), empty=torch.from_numpy(empty).to(device),
                      max_cache_length=int(lens.max()) if B else 0, first_page=first, num_keys=keys)


def decode_local(q, blocks, scales, shard: LocalShard, layer_idx: int, softmax_scale: float, stream=None):
    """This rank's part: the ordinary decode over its key ranges (q_len 1), lse = -inf where empty."""
    if q.shape[1] != 1:
        raise ValueError("context parallelism here takes one query token per request")
    out, lse = _lib.decode(q, blocks, scales, shard.cache_lengths, shard.lookup_table, shard.scales_lookup_table,
                           1, shard.max_cache_length, layer_idx, softmax_scale, stream=stream)
    if bool(shard.empty.any()):
        lse.masked_fill_(shard.empty.view(-1, 1, 1), float("-inf"))
    return out, lse


def exchange_parts(out, lse, group=None):
    """All-gather of every rank's (out, lse) into [world, ...] tensors, ordered by rank (NCCL's
    all_gather_into_tensor on GPUs; the list form elsewhere)."""
    import torch.distributed as dist
    world = dist.get_world_size(group)
    out, lse = out.contiguous(), lse.contiguous()
    if out.is_cuda:
        outs = torch.empty((world,) + tuple(out.shape), dtype=out.dtype, device=out.device)
        lses = torch.empty((world,) + tuple(lse.shape), dtype=lse.dtype, device=lse.device)
        dist.all_gather_into_tensor(outs, out, group=group)
        dist.all_gather_into_tensor(lses, lse, group=group)
        return outs, lses
    ol = [torch.empty_like(out) for _ in range(world)]
    ll = [torch.empty_like(lse) for _ in range(world)]
    dist.all_gather(ol, out, group=group)
    dist.all_gather(ll, lse, group=group)
    return torch.stack(ol), torch.stack(ll)


def decode_context_parallel(q, blocks, scales, shard: LocalShard, layer_idx: int, softmax_scale: float,
                            group=None, stream=None):
    """The whole step on every rank: local decode, exchange of (out, lse), LSE merge."""
    out, lse = decode_local(q, blocks, scales, shard, layer_idx, softmax_scale, stream=stream)
    outs, lses = exchange_parts(out, lse, group)
    return _lib.merge_parts(outs, lses, stream=stream)
