"""Decode of long sequences split along the cache across the ranks of a
process group (one process per GPU).

The attention of a decode step is one softmax over the rows of
[representatives || window] ("Latent-Condensed Transformer for Efficient
Long Context Modeling", 整体框架).  Cut those rows into shards, and each
shard gives the output normalised over its own rows plus the log-sum-exp of
its logits; merging by log-sum-exp restores the whole softmax exactly.  Each
rank holds a contiguous run of whole groups of every sequence's cache (the
last rank also holds the window).  It computes its shard record with
lca_decode_shard, the records are all-gathered (16 * 513 floats, about
33 KB, per sequence and rank), and every rank merges them with
lca_combine_shards.

The only exchange is that gather.  Condensation needs no communication: a
group's representative depends on its own rows and on the summary query,
which every rank holds.
"""
from __future__ import annotations

import torch
import torch.distributed as dist

from . import api


def shard_bounds(L: int, n: int, g: int = 16, w: int = 1024) -> list[tuple[int, int]]:
    """Row ranges [row0, row1) of n shards of a cache of length L.  Cuts fall
    on multiples of g inside the condensed history (rows below m*g, with
    m = max(0, floor((L - w) / g))), so every shard holds whole groups and
    the last one holds the whole window.  Shards are balanced by rows, since
    each row is read once.  Every shard is non-empty; raises ValueError when
    there are too few groups for n shards."""
    if n < 1 or L < 1 or g < 1 or w < 0:
        raise ValueError("need n >= 1, L >= 1, g >= 1, w >= 0")
    m = max(0, (L - w) // g)
    # the last cut leaves at least one row to the last shard
    hi = m * g if L > m * g else (m - 1) * g
    if n > 1 and hi < (n - 1) * g:
        raise ValueError(f"L={L} has {m} groups: too few for {n} shards")
    cuts: list[int] = []
    for r in range(1, n):
        c = int(round(r * L / n / g)) * g
        c = max(c, cuts[-1] + g if cuts else g)
        c = min(c, hi - (n - 1 - r) * g)
        cuts.append(c)
    return list(zip([0] + cuts, cuts + [L]))


def split_l_decode(cache_shard, q_recent, q, w_uv, L: int, row0: int, *, g: int = 16, w: int = 1024,
                   scale=None, group=None, out=None, ws=None, shard_fn=None, combine_fn=None):
    """One decode step of B sequences whose caches are split across the
    ranks of `group`.  This rank holds rows row0 .. row0 + L_shard - 1 of
    every sequence (cache_shard [B, L_shard, 576], packed or a view into a
    larger buffer such as full[:, row0:row1]); q_recent and q are the
    same on every rank.  Returns out [B, 16, 128] (the same on every rank).
    Without an initialised process group (or with one rank) the shard is
    the whole cache and no exchange takes place.

    shard_fn and combine_fn default to the library's lca_decode_shard and
    lca_combine_shards."""
    shard_fn = api.lca_decode_shard if shard_fn is None else shard_fn
    combine_fn = api.lca_combine_shards if combine_fn is None else combine_fn
    B = q.shape[0]
    part = shard_fn(cache_shard, q_recent, q, L, row0, g=g, w=w, scale=scale, ws=ws)
    if not dist.is_initialized() or dist.get_world_size(group) == 1:
        return combine_fn(part.view(1, part.numel()), w_uv, B, out=out)
    n = dist.get_world_size(group)
    parts = part.new_empty(n * part.numel())
    dist.all_gather_into_tensor(parts, part, group=group)
    return combine_fn(parts.view(n, part.numel()), w_uv, B, out=out)
