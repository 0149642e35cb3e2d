"""CPU oracle for MLA decode and latent-condensed attention (LCA).

TEST INFRASTRUCTURE ONLY.  The CUDA library and its Python binding never
import this package.  Only the tests, the package smoke check and the
benchmark's CPU-baseline / reference leg use it.

The arithmetic lives in ``lca_oracle.c`` (plain fp64 loops, one function per
definition of "Latent-Condensed Transformer for Efficient Long Context
Modeling", sections 整体框架 / 关键设计 1-3).  This module compiles it with
gcc (OpenMP over independent sequences, groups, heads or prefill blocks) and
exposes numpy wrappers.  Inputs are the exact bf16 bit patterns (uint16
arrays); outputs are fp64.
"""
from __future__ import annotations

import ctypes
import os
import subprocess

import numpy as np

_HERE = os.path.dirname(os.path.abspath(__file__))
_SRC = os.path.join(_HERE, "lca_oracle.c")
_LIB = os.path.join(_HERE, "liblca_oracle.so")
_lib = None


def build(force: bool = False) -> str:
    """Compile the oracle shared library (gcc -O2 -fopenmp, no fast-math)."""
    if force or not os.path.exists(_LIB) or os.path.getmtime(_LIB) < os.path.getmtime(_SRC):
        tmp = _LIB + f".tmp{os.getpid()}"
        subprocess.check_call(["gcc", "-O2", "-fopenmp", "-fPIC", "-shared", "-std=c11",
                               "-o", tmp, _SRC, "-lm"])
        os.replace(tmp, _LIB)
    return _LIB


def _load():
    global _lib
    if _lib is None:
        build()
        lib = ctypes.CDLL(_LIB)
        P = ctypes.c_void_p
        I = ctypes.c_int
        Lg = ctypes.c_long
        Dd = ctypes.c_double
        lib.ora_num_threads.restype = I
        lib.ora_num_groups.restype = Lg
        lib.ora_num_groups.argtypes = [Lg, I, I]
        lib.ora_lca_condense_fv.restype = I
        lib.ora_lca_condense_fv.argtypes = [P, P, I, Lg, I, I, I, I, I, Dd, I, P, P, P, P, P, P]
        lib.ora_mla_decode.restype = I
        lib.ora_mla_decode.argtypes = [P, P, P, I, Lg, I, I, I, I, Dd, P, P]
        lib.ora_lca_decode_f.restype = I
        lib.ora_lca_decode_f.argtypes = [P, P, P, P, I, Lg, I, I, I, I, I, I, Dd, P, P, P, P]
        lib.ora_lca_attend_reps.restype = I
        lib.ora_lca_attend_reps.argtypes = [P, P, P, P, I, Lg, I, I, I, I, I, I, Dd, P, P]
        lib.ora_lca_decode_stored_f.restype = I
        lib.ora_lca_decode_stored_f.argtypes = [P, P, P, I, Lg, I, I, I, I, I, I, Dd, P, P, P, P]
        lib.ora_lca_decode_shard_f.restype = I
        lib.ora_lca_decode_shard_f.argtypes = [P, P, P, I, Lg, I, I, I, I, I, Dd, Lg, Lg, P, P, P,
                                               P]
        lib.ora_lca_prefill_fv.restype = I
        lib.ora_lca_prefill_fv.argtypes = [P, P, P, I, Lg, Lg, Lg, I, I, I, I, I, I, Dd, I, P, Lg,
                                           P, P, P, P]
        _lib = lib
    return _lib


def _u16(a):
    a = np.ascontiguousarray(a)
    assert a.dtype == np.uint16, a.dtype
    return a


def _bf16_to_f64(a):
    """Exact widening of bf16 bit patterns (the high half of an fp32)."""
    return (a.astype(np.uint32) << 16).view(np.float32).astype(np.float64)


def _ptr(a):
    return None if a is None else a.ctypes.data_as(ctypes.c_void_p)


def _forced(anchor_in, shape):
    """Forced anchors (absolute positions) as a contiguous int32 array of
    `shape`, or None."""
    if anchor_in is None:
        return None
    a = np.ascontiguousarray(np.asarray(anchor_in, dtype=np.int32))
    if a.shape != tuple(shape):
        raise ValueError(f"anchor_in has shape {a.shape}, expected {tuple(shape)}")
    return a


def _check_forced(rc):
    if rc == -2:
        raise ValueError("a forced anchor lies outside its group")
    if rc != 0:
        raise ValueError(f"oracle call failed ({rc})")


def num_threads() -> int:
    return _load().ora_num_threads()


def num_groups(L: int, g: int, w: int) -> int:
    """m = max(0, floor((L - w) / g))."""
    return int(_load().ora_num_groups(L, g, w))


# condensation variants: the method and the two ablations (pool the RoPE key
# too; keep only the most important token)
LCA, POOL_POSITION, SPARSE = 0, 1, 2


def lca_condense(cache, q_recent, g: int, w: int, scale: float, dr: int = 64, variant: int = LCA,
                 anchor_in=None):
    """cache [B,L,dc+dr] u16, q_recent [B,g,H,dc+dr] u16 ->
    dict(rep_c [B,m,dc], rep_k [B,m,dr], anchor [B,m] int32 (position in the
    sequence), alpha [B,m,g], score [B,m,g]).  anchor_in [B,m] (absolute
    positions) forces the anchors instead of the argmax ("forced-anchor"
    mode, for checking a result computed with another valid anchor where the
    group maximum is a near-tie); nothing else changes."""
    cache, q_recent = _u16(cache), _u16(q_recent)
    B, L, D = cache.shape
    H = q_recent.shape[2]
    dc = D - dr
    m = num_groups(L, g, w)
    out = dict(rep_c=np.zeros((B, m, dc)), rep_k=np.zeros((B, m, dr)),
               anchor=np.zeros((B, m), np.int32), alpha=np.zeros((B, m, g)),
               score=np.zeros((B, m, g)))
    forced = _forced(anchor_in, (B, m))
    _check_forced(_load().ora_lca_condense_fv(
        _ptr(cache), _ptr(q_recent), B, L, H, dc, dr, g, w, scale, int(variant), _ptr(forced),
        _ptr(out["rep_c"]), _ptr(out["rep_k"]), _ptr(out["anchor"]), _ptr(out["alpha"]),
        _ptr(out["score"])))
    return out


def mla_decode(cache, q, w_uv, scale: float, dr: int = 64):
    """-> (o_lat [B,H,dc], out [B,H,dv]) in fp64."""
    cache, q, w_uv = _u16(cache), _u16(q), _u16(w_uv)
    B, L, D = cache.shape
    H = q.shape[1]
    dc = D - dr
    dv = w_uv.shape[2]
    o_lat = np.zeros((B, H, dc))
    out = np.zeros((B, H, dv))
    _load().ora_mla_decode(_ptr(cache), _ptr(q), _ptr(w_uv), B, L, H, dc, dr, dv, scale,
                           _ptr(o_lat), _ptr(out))
    return o_lat, out


def lca_decode(cache, q_recent, q, w_uv, g: int, w: int, scale: float, dr: int = 64,
               anchor_in=None):
    """-> (o_lat [B,H,dc], out [B,H,dv], anchor [B,m]).  anchor_in [B,m]:
    forced anchors (see lca_condense)."""
    cache, q_recent, q, w_uv = _u16(cache), _u16(q_recent), _u16(q), _u16(w_uv)
    B, L, D = cache.shape
    H = q.shape[1]
    dc = D - dr
    dv = w_uv.shape[2]
    m = num_groups(L, g, w)
    o_lat = np.zeros((B, H, dc))
    out = np.zeros((B, H, dv))
    anchor = np.zeros((B, max(m, 1)), np.int32)
    forced = _forced(anchor_in, (B, m))
    _check_forced(_load().ora_lca_decode_f(_ptr(cache), _ptr(q_recent), _ptr(q), _ptr(w_uv), B, L,
                                           H, dc, dr, dv, g, w, scale, _ptr(forced), _ptr(o_lat),
                                           _ptr(out), _ptr(anchor)))
    return o_lat, out, anchor[:, :m]


def lca_decode_shard(cache, q_recent, q, g: int, w: int, scale: float, row0: int, row1: int,
                     dr: int = 64, anchor_in=None):
    """One shard (rows row0 .. row1-1) of the LCA decode attention.
    -> (o [B,H,dc] normalised over the shard's rows, lse [B,H] = natural
    log-sum-exp of the shard's logits, anchor [B,m_shard] absolute).
    anchor_in [B,m] (every group of the sequence, absolute): forced anchors."""
    cache, q_recent, q = _u16(cache), _u16(q_recent), _u16(q)
    B, L, D = cache.shape
    H = q.shape[1]
    dc = D - dr
    m = num_groups(L, g, w)
    m_shard = max(0, (min(row1, m * g) - row0) // g)
    o = np.zeros((B, H, dc))
    lse = np.zeros((B, H))
    anchor = np.zeros((B, max(m_shard, 1)), np.int32)
    forced = _forced(anchor_in, (B, m))
    rc = _load().ora_lca_decode_shard_f(_ptr(cache), _ptr(q_recent), _ptr(q), B, L, H, dc, dr, g,
                                        w, scale, row0, row1, _ptr(forced), _ptr(o), _ptr(lse),
                                        _ptr(anchor))
    if rc == -1:
        raise ValueError("shard rows must start at a group boundary and be non-empty")
    _check_forced(rc)
    return o, lse, anchor[:, :m_shard]


def combine_shards(o_parts, lse_parts, w_uv):
    """Merge attention outputs over disjoint row sets: with S = log sum_s
    exp(lse_s), o = sum_s exp(lse_s - S) o_s (each o_s normalised over its
    rows), then the per-head W_UV up-projection out_h = W_UV[h]^T o_h.
    o_parts [n,B,H,dc], lse_parts [n,B,H] -> (o_lat [B,H,dc], out [B,H,dv])."""
    o_parts, lse_parts = np.asarray(o_parts, np.float64), np.asarray(lse_parts, np.float64)
    top = lse_parts.max(axis=0)
    wts = np.exp(lse_parts - top)                        # [n,B,H]
    o_lat = (wts[..., None] * o_parts).sum(axis=0) / wts.sum(axis=0)[..., None]
    wv = _bf16_to_f64(_u16(w_uv))                        # [H,dc,dv]
    out = np.einsum("bhk,hkv->bhv", o_lat, wv)
    return o_lat, out


def lca_attend_reps(cache, rep, q, w_uv, g: int, w: int, scale: float, dr: int = 64):
    """Attention over bf16 representative rows rep [B,m,dc+dr] + window.
    -> (o_lat, out)."""
    cache, rep, q, w_uv = _u16(cache), _u16(rep), _u16(q), _u16(w_uv)
    B, L, D = cache.shape
    H = q.shape[1]
    dc = D - dr
    dv = w_uv.shape[2]
    o_lat = np.zeros((B, H, dc))
    out = np.zeros((B, H, dv))
    _load().ora_lca_attend_reps(_ptr(cache), _ptr(rep), _ptr(q), _ptr(w_uv), B, L, H, dc, dr,
                                dv, g, w, scale, _ptr(o_lat), _ptr(out))
    return o_lat, out


def lca_decode_stored(cache, q_all, w_uv, g: int, w: int, scale: float, dr: int = 64,
                      anchor_in=None):
    """Stored-representative decode at cache length L: group j condensed with
    the summary query of the step where it left the window (queries at
    positions w + g j .. w + g j + g - 1), query at L-1 attends [reps || window].
    q_all [B,L,H,D] u16.  -> (o_lat [B,H,dc], out [B,H,dv], anchor [B,m]).
    anchor_in [B,m]: forced anchors (see lca_condense)."""
    cache, q_all, w_uv = _u16(cache), _u16(q_all), _u16(w_uv)
    B, L, D = cache.shape
    H = q_all.shape[2]
    dc = D - dr
    dv = w_uv.shape[2]
    m = num_groups(L, g, w)
    o_lat = np.zeros((B, H, dc))
    out = np.zeros((B, H, dv))
    anchor = np.zeros((B, max(m, 1)), np.int32)
    forced = _forced(anchor_in, (B, m))
    _check_forced(_load().ora_lca_decode_stored_f(_ptr(cache), _ptr(q_all), _ptr(w_uv), B, L, H,
                                                  dc, dr, dv, g, w, scale, _ptr(forced),
                                                  _ptr(o_lat), _ptr(out), _ptr(anchor)))
    return o_lat, out, anchor[:, :m]


def lca_prefill(cache, qpre, w_uv, q_start: int, q_len: int, g: int, w: int, scale: float,
                blocks=None, dr: int = 64, want_anchor: bool = False, want_olat: bool = True,
                variant: int = LCA, anchor_in=None):
    """Blockwise LCA prefill.  -> (o_lat [B,q_len,H,dc] | None, out [B,q_len,H,dv], anchor|None).
    `blocks` = absolute block indices to evaluate (others left as NaN).
    `variant`: the method (LCA) or an ablation (POOL_POSITION, SPARSE).
    anchor_in [B, q_len/g, max(1, m_last)] (laid out like the anchor output;
    entries of groups a block does not have are ignored): forced anchors of
    the evaluated blocks (see lca_condense)."""
    cache, qpre, w_uv = _u16(cache), _u16(qpre), _u16(w_uv)
    B, L, D = cache.shape
    H = qpre.shape[2]
    dc = D - dr
    dv = w_uv.shape[2]
    o_lat = np.full((B, q_len, H, dc), np.nan) if want_olat else None
    out = np.full((B, q_len, H, dv), np.nan)
    bl = None
    nbl = 0
    if blocks is not None:
        bl = np.ascontiguousarray(np.asarray(blocks, dtype=np.int64))
        nbl = len(bl)
    m_max = num_groups(q_start + q_len - g, g, w)
    anchor = np.full((B, q_len // g, max(m_max, 1)), -1, np.int32) if want_anchor else None
    forced = _forced(anchor_in, (B, q_len // g, max(m_max, 1)))
    rc = _load().ora_lca_prefill_fv(_ptr(cache), _ptr(qpre), _ptr(w_uv), B, L, q_start, q_len, H,
                                    dc, dr, dv, g, w, scale, int(variant), _ptr(bl), nbl,
                                    _ptr(forced), _ptr(o_lat), _ptr(out), _ptr(anchor))
    if rc == -1:
        raise ValueError("bad prefill range")
    _check_forced(rc)
    return o_lat, out, anchor
