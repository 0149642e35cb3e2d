"""Seeded synthetic inputs for MLA / LCA decode and prefill.

This module is shared by the CUDA path's tests, the benchmark and the CPU
oracle's tests.  It holds none of the attention arithmetic: it only draws
tensors and lays them out the way an MLA latent KV cache stores them.

Recipe (every tensor bf16, rounded to nearest-even from fp32/fp64):

* cache row = [ c^KV (512) | k^R (64) ], 1152 bytes per token, one
  contiguous [B, L, 576] tensor.  c^KV ~ N(0, 1).  k^R is drawn ~ N(0, 1)
  and then rotated by RoPE (base 10000) at its own absolute position, in
  fp64, before rounding: the cache holds keys that are already rotated, as an
  MLA cache does (the decoupled RoPE key of "Latent-Condensed Transformer for
  Efficient Long Context Modeling", 研究背景与动机 / 关键设计 2).  Pairs are
  interleaved (2k, 2k+1) with theta_k = 10000^(-2k/64).
* absorbed decode query q[B, 16, 576] ~ N(0, 1)/sqrt(576)  (latent part
  q_lat = W_UK^T q_nope and an already-rotated rope part).
* recent queries q_recent[B, g, 16, 576] ~ N(0, 1)/sqrt(576); the last one
  is the current query, so q_recent[:, g-1] == q.
* W_UV[16, 512, 128] ~ N(0, 1/512).
* prefill queries q[B, L, 16, 576] ~ N(0, 1)/sqrt(576).

Draw order for one generator seeded with `seed`: for each sequence b in
order, c^KV[b] then raw k^R[b]; then q, then q_recent (g-1 older queries;
the current query is appended), then W_UV.  `peak` multiplies every query
(test-only "peaked" variant that makes pooling weights and anchors far from
uniform).
"""
from __future__ import annotations

import math
from dataclasses import dataclass

import torch

H = 16          # heads
D_C = 512       # latent width (c^KV)
D_R = 64        # decoupled RoPE key width (k^R)
D = D_C + D_R   # cache row width, 576
D_V = 128       # per-head value width after W_UV
ROPE_BASE = 10000.0


def default_scale() -> float:
    """Softmax scale 1/sqrt(128 + 64): the per-head q.k width of the
    decompressed MLA head (128 nope + 64 rope)."""
    return 1.0 / math.sqrt(192.0)


def rope_rotate_(k: torch.Tensor, pos0: int) -> torch.Tensor:
    """Rotate raw keys k[n, 64] (fp64, in place) at positions pos0..pos0+n-1."""
    n, dr = k.shape
    half = dr // 2
    inv = ROPE_BASE ** (-torch.arange(half, dtype=torch.float64) * 2.0 / dr)
    pos = torch.arange(pos0, pos0 + n, dtype=torch.float64)
    ang = pos[:, None] * inv[None, :]
    cos, sin = torch.cos(ang), torch.sin(ang)
    x0 = k[:, 0::2].clone()
    x1 = k[:, 1::2].clone()
    k[:, 0::2] = x0 * cos - x1 * sin
    k[:, 1::2] = x0 * sin + x1 * cos
    return k


def make_cache(gen: torch.Generator, B: int, L: int) -> torch.Tensor:
    """[B, L, 576] bf16 latent cache drawn in the documented order."""
    cache = torch.empty(B, L, D, dtype=torch.bfloat16)
    chunk = 1 << 16
    for b in range(B):
        c = torch.randn(L, D_C, generator=gen, dtype=torch.float32)
        cache[b, :, :D_C] = c.to(torch.bfloat16)
        del c
        kr = torch.randn(L, D_R, generator=gen, dtype=torch.float32)
        for s in range(0, L, chunk):
            e = min(L, s + chunk)
            k64 = kr[s:e].to(torch.float64)
            rope_rotate_(k64, s)
            cache[b, s:e, D_C:] = k64.to(torch.bfloat16)
        del kr
    return cache


@dataclass
class DecodeInputs:
    cache: torch.Tensor      # [B, L, 576] bf16
    q: torch.Tensor          # [B, 16, 576] bf16 (current query)
    q_recent: torch.Tensor   # [B, g, 16, 576] bf16 (q_recent[:, g-1] == q)
    w_uv: torch.Tensor       # [16, 512, 128] bf16
    B: int
    L: int
    g: int
    w: int
    scale: float


def make_decode_inputs(B: int, L: int, g: int = 16, w: int = 1024, seed: int = 0,
                       peak: float = 1.0) -> DecodeInputs:
    gen = torch.Generator().manual_seed(seed)
    cache = make_cache(gen, B, L)
    qs = peak / math.sqrt(D)
    q = (torch.randn(B, H, D, generator=gen) * qs).to(torch.bfloat16)
    older = (torch.randn(B, g - 1, H, D, generator=gen) * qs).to(torch.bfloat16)
    q_recent = torch.cat([older, q[:, None]], dim=1).contiguous()
    w_uv = (torch.randn(H, D_C, D_V, generator=gen) / math.sqrt(D_C)).to(torch.bfloat16)
    return DecodeInputs(cache, q, q_recent, w_uv, B, L, g, w, default_scale())


@dataclass
class PrefillInputs:
    cache: torch.Tensor   # [B, L, 576] bf16
    q: torch.Tensor       # [B, L, 16, 576] bf16
    w_uv: torch.Tensor    # [16, 512, 128] bf16
    B: int
    L: int
    g: int
    w: int
    scale: float


def make_prefill_inputs(B: int, L: int, g: int = 16, w: int = 1024, seed: int = 0,
                        peak: float = 1.0) -> PrefillInputs:
    gen = torch.Generator().manual_seed(seed)
    cache = make_cache(gen, B, L)
    qs = peak / math.sqrt(D)
    q = torch.empty(B, L, H, D, dtype=torch.bfloat16)
    chunk = 1 << 14
    for b in range(B):
        for s in range(0, L, chunk):
            e = min(L, s + chunk)
            q[b, s:e] = (torch.randn(e - s, H, D, generator=gen) * qs).to(torch.bfloat16)
    w_uv = (torch.randn(H, D_C, D_V, generator=gen) / math.sqrt(D_C)).to(torch.bfloat16)
    return PrefillInputs(cache, q, w_uv, B, L, g, w, default_scale())


def bf16_bits(t: torch.Tensor):
    """uint16 numpy view of a contiguous bf16 tensor (the exact stored bits)."""
    assert t.dtype == torch.bfloat16
    return t.contiguous().view(torch.int16).numpy().view("uint16")


# Named workloads: shapes of the decode / prefill cases the kernels are
# measured and checked on.
WORKLOADS = {
    "decode_b1_l4k":    dict(kind="decode", B=1, L=4096),
    "decode_b32_l32k":  dict(kind="decode", B=32, L=32768),
    "decode_b8_l128k":  dict(kind="decode", B=8, L=131072),
    "prefill_b1_l128k": dict(kind="prefill", B=1, L=131072),
    "decode_b1_l1m":    dict(kind="decode", B=1, L=1048576),
    # smaller cases for profiler captures (cache 302 MB / queries 302 MB, > L2)
    "decode_b8_l32k":   dict(kind="decode", B=8, L=32768),
    "prefill_b1_l16k":  dict(kind="prefill", B=1, L=16384),
}
