"""Inputs with planted argmax near-ties (test input construction only; no
attention arithmetic).

In a planted group two adjacent rows i0, i1 = i0 + 1 are the group's top
two candidates and differ in their latent only at one coordinate k*, where
i0 holds 0 and i1 holds sign(u_k*) * 2^-30, u being the (fp64) summary
vector of the importance score.  Their importance scores then differ by
|u_k*| * 2^-30 (~1e-13, far below fp32 resolution of the scores ~1e-10):
the fp64 oracle picks i1, a GPU computing the scores in fp32 sees a tie and
takes the first index i0.  Both are valid anchors under the near-tie rule.

So that the choice matters, the two rows carry very different RoPE keys in
dims 32..63, and those dims are made invisible to the importance score: the
recent queries come in pairs whose RoPE dims 32..63 cancel exactly, so the
exact summary query is zero there (an fp32 sum in another order may keep a
residual of a few ulps), while every individual query still sees the keys in
its attention logits.
"""
from __future__ import annotations

import torch

from mla_latent_space_lca_b200.inputs import D_C

G = 16
TINY = 2.0 ** -30
HALF = D_C + 32          # first RoPE dim hidden from the importance score
KEY_SCALE = 32.0


def _cancel_pairs(q, dim):
    """q[..., t, ..., HALF:] of the odd slots along `dim` := minus the even
    slot before it."""
    n = q.shape[dim]
    for t in range(0, n - 1, 2):
        src = q.select(dim, t)[..., HALF:]
        q.select(dim, t + 1)[..., HALF:] = -src


def plant_decode(inp, n_groups: int, seed: int, w: int = 1024):
    """Decode inputs (inputs.make_decode_inputs) -> (cache, q_recent, q,
    planted [(b, j)]) with near-ties planted in n_groups groups of every
    sequence.  q_recent[:, g-1] stays equal to q."""
    gen = torch.Generator().manual_seed(seed)
    cache, q_recent = inp.cache.clone(), inp.q_recent.clone()
    B, L = inp.B, inp.L
    m = max(0, (L - w) // G) if L >= w else 0
    _cancel_pairs(q_recent, 1)
    q = q_recent[:, G - 1].clone()
    # direction of the importance score (positive factor scale/H dropped)
    u = q_recent.double().sum(dim=(1, 2))                    # [B, 576]
    assert torch.all(u[:, HALF:] == 0)
    # keys that the attention sees: the current query's RoPE dims 32..63
    v = torch.sign(q[:, :, HALF:].double().sum(dim=1))       # [B, 32]
    v[v == 0] = 1
    planted = []
    for b in range(B):
        ub = u[b, :D_C]
        kstar = int(torch.argmax(ub.abs()))
        groups = torch.randperm(m, generator=gen)[:n_groups].tolist()
        for j in groups:
            o = int(torch.randint(0, G - 1, (1,), generator=gen))
            i0 = j * G + o
            x = torch.sign(ub) * torch.randn(D_C, generator=gen, dtype=torch.float64).abs() * 1.5
            x[kstar] = 0.0
            row = torch.empty(576, dtype=torch.float64)
            row[:D_C] = x
            row[D_C:HALF] = torch.randn(32, generator=gen, dtype=torch.float64)
            # which of the pair carries +v is random per group: a GPU whose
            # summary vector keeps an fp32 residual in the hidden dims then
            # breaks the tie differently from group to group
            sg = 1.0 if float(torch.rand(1, generator=gen)) < 0.5 else -1.0
            row[HALF:] = sg * KEY_SCALE * v[b]
            cache[b, i0] = row.to(torch.bfloat16)
            row[HALF:] = -sg * KEY_SCALE * v[b]
            row[kstar] = float(torch.sign(ub[kstar])) * TINY
            cache[b, i0 + 1] = row.to(torch.bfloat16)
            planted.append((b, j))
    return cache, q_recent, q, planted


def plant_prefill(inp, n_groups: int, seed: int):
    """Prefill inputs (inputs.make_prefill_inputs) -> (cache, q, planted
    group indices).  Every block's queries cancel in RoPE dims 32..63 in
    pairs, so each block's summary query is zero there.  The planted rows
    have random latents of three times the usual size: in roughly half of
    the blocks they are the group's top two, and there the fp64 order of
    the pair follows the sign of that block's u_k* (k* = 0)."""
    gen = torch.Generator().manual_seed(seed)
    cache, q = inp.cache.clone(), inp.q.clone()
    B, L = inp.B, inp.L
    qv = q.view(B, L // G, G, 16, 576)
    _cancel_pairs(qv, 2)
    n_hist = L // G
    groups = torch.randperm(max(1, n_hist // 2), generator=gen)[:n_groups].tolist()
    for b in range(B):
        for j in groups:
            o = int(torch.randint(0, G - 1, (1,), generator=gen))
            i0 = j * G + o
            row = torch.empty(576, dtype=torch.float64)
            row[:D_C] = torch.randn(D_C, generator=gen, dtype=torch.float64) * 3.0
            row[0] = 0.0
            row[D_C:HALF] = torch.randn(32, generator=gen, dtype=torch.float64)
            sgn = torch.sign(torch.randn(32, generator=gen, dtype=torch.float64))
            row[HALF:] = KEY_SCALE * sgn
            cache[b, i0] = row.to(torch.bfloat16)
            row[HALF:] = -KEY_SCALE * sgn
            row[0] = TINY
            cache[b, i0 + 1] = row.to(torch.bfloat16)
    return cache, q, groups
