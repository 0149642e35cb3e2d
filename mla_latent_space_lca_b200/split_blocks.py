"""Blockwise prefill of one prompt split over the ranks of a process group,
one process per GPU.

Every query block of the prefill is independent given the cache. Block k
condenses its own history with its own summary query and attends its own
representatives and causal window (the blockwise prefill of "Latent-Condensed
Transformer for Efficient Long Context Modeling", 整体框架 and 关键设计
1-3). Each rank therefore runs lca_prefill_block over a contiguous range of
blocks, with the cache replicated, and writes its own rows of the output. No
exchange is needed in the data path.

Later blocks attend more representatives and condense more history, so the
ranges are balanced by work, not by block count.
"""
from __future__ import annotations


def block_flops(k: int, g: int = 16, w: int = 1024) -> int:
    """Algorithmic flops of prefill block k.

    Let m = max(0, k - ceil(w/g)). The block's g queries attend m
    representatives plus their causal window. Every history row is scored and
    pooled for the condensation. W_UV up-projects each query.
    """
    cw = -(-w // g)
    m = max(0, k - cw)
    keys = g * m + sum(g * k + t - g * m + 1 for t in range(g))
    att = keys * 16 * (576 + 512) * 2
    cond = g * m * (576 + 512) * 2
    wuv = g * 16 * 512 * 128 * 2
    return att + cond + wuv


def prefill_block_ranges(L: int, n: int, g: int = 16, w: int = 1024) -> list[tuple[int, int]]:
    """(q_start, q_len) of n contiguous ranges covering the floor(L/g) whole
    blocks of [0, L), cut where the cumulative work crosses i/n of the total.
    Every range is non-empty when there are at least n blocks (raises
    ValueError otherwise)."""
    nb = L // g
    if n < 1 or nb < n:
        raise ValueError(f"{nb} blocks cannot be split over {n} ranks")
    cost = [block_flops(k, g, w) for k in range(nb)]
    total = float(sum(cost))
    cuts, acc, r = [], 0.0, 1
    for k in range(nb):
        acc += cost[k]
        while r < n and acc >= total * r / n:
            cuts.append(k + 1)
            r += 1
    # keep every range non-empty and every cut inside (0, nb)
    for i in range(len(cuts)):
        lo = (cuts[i - 1] + 1) if i else 1
        hi = nb - (n - 1 - i)
        cuts[i] = min(max(cuts[i], lo), hi)
    bounds = [0] + cuts + [nb]
    return [(g * a, g * (b - a)) for a, b in zip(bounds[:-1], bounds[1:])]
