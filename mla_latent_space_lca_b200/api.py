"""PyTorch-facing wrappers of the C ABI (argument marshalling only).

Every function takes CUDA tensors, checks dtype / shape / contiguity,
allocates missing outputs and scratch with torch (device memory is the only
thing PyTorch provides here), and calls the corresponding entry point of
liblca_b200.so on the current stream.  All arithmetic runs in the library's
kernels.
"""
from __future__ import annotations

import ctypes
import math

import torch

from . import _lib
from ._lib import LcaParams, check

H, D_C, D_R, D, D_V = 16, 512, 64, 576, 128


def default_scale() -> float:
    return 1.0 / math.sqrt(192.0)


def _params(g: int, w: int, scale: float | None, variant: int = 0, pitch: int = 0) -> LcaParams:
    return LcaParams(int(g), int(w), float(default_scale() if scale is None else scale), int(variant),
                     int(pitch))


def _ptr(t):
    return None if t is None else ctypes.c_void_p(t.data_ptr())


def _stream(stream=None):
    s = stream if stream is not None else torch.cuda.current_stream()
    return ctypes.c_void_p(s.cuda_stream)


def _need(t, name, dtype, shape=None, host=False):
    """A contiguous tensor of this dtype (and shape) on the GPU, or, with
    host=True, in pinned host memory (read or written in place by the
    kernels over the host link)."""
    if not isinstance(t, torch.Tensor):
        raise TypeError(f"{name} must be a tensor")
    if not t.is_cuda and not (host and t.is_pinned()):
        raise TypeError(f"{name} must be a CUDA tensor" + (" or pinned host memory" if host else ""))
    if t.dtype != dtype:
        raise TypeError(f"{name} must be {dtype}, got {t.dtype}")
    if not t.is_contiguous():
        raise ValueError(f"{name} must be contiguous")
    if shape is not None and tuple(t.shape) != tuple(shape):
        raise ValueError(f"{name} has shape {tuple(t.shape)}, expected {tuple(shape)}")


def _cache(t, name="cache"):
    """A cache tensor [B, L, 576] bf16, either packed or rows 0 .. L-1 of each
    sequence of a larger [B, L_max, 576] buffer (a view such as
    buf[:, :L]).  Returns the pitch in rows to pass to the library (0 when
    packed)."""
    if not isinstance(t, torch.Tensor) or not t.is_cuda:
        raise TypeError(f"{name} must be a CUDA tensor")
    if t.dtype != torch.bfloat16:
        raise TypeError(f"{name} must be torch.bfloat16, got {t.dtype}")
    if t.dim() != 3 or t.shape[2] != D:
        raise ValueError(f"{name} has shape {tuple(t.shape)}, expected (B, L, {D})")
    if t.is_contiguous():
        return 0
    B, L, _ = t.shape
    s0, s1, s2 = t.stride()
    if s2 != 1 or s1 != D or s0 % D or s0 < L * D:
        raise ValueError(f"{name} must hold each sequence's rows contiguously (strides {t.stride()})")
    return s0 // D


def num_groups(L: int, g: int = 16, w: int = 1024) -> int:
    return int(_lib.lib().lca_num_groups(L, _params(g, w, None)))


def workspace_bytes(op: int, B: int, L: int, q_len: int = 0, g: int = 16, w: int = 1024) -> int:
    return int(_lib.lib().lca_workspace_bytes(op, B, L, q_len, _params(g, w, None)))


def workspace(op: int, B: int, L: int, q_len: int = 0, g: int = 16, w: int = 1024,
              device=None) -> torch.Tensor:
    n = workspace_bytes(op, B, L, q_len, g, w)
    return torch.empty(max(n, 256), dtype=torch.uint8, device=device or "cuda")


def mla_decode_attn(cache, q, w_uv, scale=None, out=None, o_lat=None, ws=None, stream=None):
    B, L, _ = cache.shape
    pitch = _cache(cache)
    _need(q, "q", torch.bfloat16, (B, H, D))
    _need(w_uv, "w_uv", torch.bfloat16, (H, D_C, D_V))
    out = torch.empty(B, H, D_V, dtype=torch.float32, device=cache.device) if out is None else out
    _need(out, "out", torch.float32, (B, H, D_V), host=True)
    if o_lat is not None:
        _need(o_lat, "o_lat", torch.float32, (B, H, D_C))
    ws = workspace(_lib.OP_MLA_DECODE, B, L, device=cache.device) if ws is None else ws
    if pitch:   # a strided cache: MLA decode through lca_decode with g = 1
        rc = _lib.lib().lca_decode(_ptr(cache), None, _ptr(q), _ptr(w_uv), B, L, _params(1, 0, scale, 0, pitch),
                                   _ptr(out), _ptr(o_lat), None, _ptr(ws), ws.numel(), _stream(stream))
        check(rc, "mla_decode_attn")
        return out
    rc = _lib.lib().mla_decode_attn(_ptr(cache), _ptr(q), _ptr(w_uv), B, L,
                                    float(default_scale() if scale is None else scale), _ptr(out),
                                    _ptr(o_lat), _ptr(ws), ws.numel(), _stream(stream))
    check(rc, "mla_decode_attn")
    return out


def lca_condense(cache, q_recent, g=16, w=1024, scale=None, rep=None, anchor=None, alpha=None,
                 ws=None, stream=None, variant=0):
    B, L, _ = cache.shape
    pitch = _cache(cache)
    _need(q_recent, "q_recent", torch.bfloat16, (B, g, H, D))
    m = num_groups(L, g, w)
    dev = cache.device
    rep = torch.empty(B, m, D, dtype=torch.bfloat16, device=dev) if rep is None else rep
    ws = workspace(_lib.OP_CONDENSE, B, L, g=g, w=w, device=dev) if ws is None else ws
    rc = _lib.lib().lca_condense(_ptr(cache), _ptr(q_recent), B, L, _params(g, w, scale, variant, pitch),
                                 _ptr(rep) if m > 0 else None, _ptr(anchor), _ptr(alpha), _ptr(ws),
                                 ws.numel(), _stream(stream))
    check(rc, "lca_condense")
    return rep


def lca_decode_attn(cache, rep, q, w_uv, g=16, w=1024, scale=None, out=None, o_lat=None, ws=None,
                    stream=None):
    B, L, _ = cache.shape
    pitch = _cache(cache)
    _need(q, "q", torch.bfloat16, (B, H, D))
    _need(w_uv, "w_uv", torch.bfloat16, (H, D_C, D_V))
    m = num_groups(L, g, w)
    if m > 0:
        _need(rep, "rep", torch.bfloat16, (B, m, D))
    out = torch.empty(B, H, D_V, dtype=torch.float32, device=cache.device) if out is None else out
    _need(out, "out", torch.float32, (B, H, D_V), host=True)
    if o_lat is not None:
        _need(o_lat, "o_lat", torch.float32, (B, H, D_C))
    ws = workspace(_lib.OP_DECODE_ATTN, B, L, g=g, w=w, device=cache.device) if ws is None else ws
    rc = _lib.lib().lca_decode_attn(_ptr(cache), _ptr(rep) if m > 0 else None, _ptr(q), _ptr(w_uv),
                                    B, L, _params(g, w, scale, 0, pitch), _ptr(out), _ptr(o_lat), _ptr(ws),
                                    ws.numel(), _stream(stream))
    check(rc, "lca_decode_attn")
    return out


def lca_condense_append(cache, q_recent, rep, j0, g=16, w=1024, scale=None, anchor=None, alpha=None,
                        ws=None, stream=None, variant=0):
    """Condense groups j0 .. m-1 into rows j0 .. of the representative cache
    rep [B, rep_cap, 576] (bf16); returns m, the number of groups now held."""
    B, L, _ = cache.shape
    pitch = _cache(cache)
    _need(q_recent, "q_recent", torch.bfloat16, (B, g, H, D))
    _need(rep, "rep", torch.bfloat16)
    if rep.dim() != 3 or rep.shape[0] != B or rep.shape[2] != D:
        raise ValueError(f"rep has shape {tuple(rep.shape)}, expected ({B}, rep_cap, {D})")
    m = num_groups(L, g, w)
    ws = workspace(_lib.OP_CONDENSE, B, L, g=g, w=w, device=cache.device) if ws is None else ws
    rc = _lib.lib().lca_condense_append(_ptr(cache), _ptr(q_recent), B, L, _params(g, w, scale, variant, pitch), int(j0),
                                        _ptr(rep), rep.shape[1], _ptr(anchor), _ptr(alpha), _ptr(ws),
                                        ws.numel(), _stream(stream))
    check(rc, "lca_condense_append")
    return m


def lca_decode_stored(cache, rep, q, w_uv, g=16, w=1024, scale=None, out=None, o_lat=None, ws=None,
                      stream=None):
    """Attention over the kept representatives rep [B, rep_cap, 576] (rows
    0 .. m-1) and the window, then W_UV."""
    B, L, _ = cache.shape
    pitch = _cache(cache)
    _need(q, "q", torch.bfloat16, (B, H, D))
    _need(w_uv, "w_uv", torch.bfloat16, (H, D_C, D_V))
    _need(rep, "rep", torch.bfloat16)
    out = torch.empty(B, H, D_V, dtype=torch.float32, device=cache.device) if out is None else out
    _need(out, "out", torch.float32, (B, H, D_V), host=True)
    if o_lat is not None:
        _need(o_lat, "o_lat", torch.float32, (B, H, D_C))
    ws = workspace(_lib.OP_DECODE_ATTN, B, L, g=g, w=w, device=cache.device) if ws is None else ws
    rc = _lib.lib().lca_decode_stored(_ptr(cache), _ptr(rep), rep.shape[1], _ptr(q), _ptr(w_uv), B, L,
                                      _params(g, w, scale, 0, pitch), _ptr(out), _ptr(o_lat), _ptr(ws), ws.numel(),
                                      _stream(stream))
    check(rc, "lca_decode_stored")
    return out


def lca_decode(cache, q_recent, q, w_uv, g=16, w=1024, scale=None, out=None, o_lat=None,
               anchor=None, ws=None, stream=None):
    B, L, _ = cache.shape
    pitch = _cache(cache)
    _need(q, "q", torch.bfloat16, (B, H, D))
    _need(w_uv, "w_uv", torch.bfloat16, (H, D_C, D_V))
    if g != 1:
        _need(q_recent, "q_recent", torch.bfloat16, (B, g, H, D))
    out = torch.empty(B, H, D_V, dtype=torch.float32, device=cache.device) if out is None else out
    _need(out, "out", torch.float32, (B, H, D_V), host=True)
    if o_lat is not None:
        _need(o_lat, "o_lat", torch.float32, (B, H, D_C))
    ws = workspace(_lib.OP_DECODE, B, L, g=g, w=w, device=cache.device) if ws is None else ws
    rc = _lib.lib().lca_decode(_ptr(cache), _ptr(q_recent), _ptr(q), _ptr(w_uv), B, L,
                               _params(g, w, scale, 0, pitch), _ptr(out), _ptr(o_lat), _ptr(anchor), _ptr(ws),
                               ws.numel(), _stream(stream))
    check(rc, "lca_decode")
    return out


def lca_decode_varlen(cache, lens, q_recent, q, w_uv, g=16, w=1024, scale=None, out=None, o_lat=None,
                      anchor=None, ws=None, stream=None):
    """Decode of a ragged batch: sequence b holds lens[b] rows (int32 CUDA
    tensor [B]) at rows 0 .. lens[b]-1 of cache [B, L, 576] (packed, or a
    view into a larger buffer); L is the largest length the buffer holds."""
    B, L, _ = cache.shape
    pitch = _cache(cache)
    _need(lens, "lens", torch.int32, (B,))
    _need(q, "q", torch.bfloat16, (B, H, D))
    _need(w_uv, "w_uv", torch.bfloat16, (H, D_C, D_V))
    if g != 1:
        _need(q_recent, "q_recent", torch.bfloat16, (B, g, H, D))
    out = torch.empty(B, H, D_V, dtype=torch.float32, device=cache.device) if out is None else out
    _need(out, "out", torch.float32, (B, H, D_V), host=True)
    if o_lat is not None:
        _need(o_lat, "o_lat", torch.float32, (B, H, D_C))
    ws = workspace(_lib.OP_DECODE, B, L, g=g, w=w, device=cache.device) if ws is None else ws
    rc = _lib.lib().lca_decode_varlen(_ptr(cache), _ptr(lens), _ptr(q_recent), _ptr(q), _ptr(w_uv), B, L,
                                      _params(g, w, scale, 0, pitch), _ptr(out), _ptr(o_lat), _ptr(anchor),
                                      _ptr(ws), ws.numel(), _stream(stream))
    check(rc, "lca_decode_varlen")
    return out


def lca_decode_stored_varlen(cache, rep, lens, q, w_uv, g=16, w=1024, scale=None, out=None, o_lat=None,
                             ws=None, stream=None):
    """Stored-representative decode of a ragged batch: sequence b holds
    lens[b] rows of cache [B, L, 576] and its first num_groups(lens[b])
    representatives in rep [B, rep_cap, 576]."""
    B, L, _ = cache.shape
    pitch = _cache(cache)
    _need(lens, "lens", torch.int32, (B,))
    _need(q, "q", torch.bfloat16, (B, H, D))
    _need(w_uv, "w_uv", torch.bfloat16, (H, D_C, D_V))
    _need(rep, "rep", torch.bfloat16)
    out = torch.empty(B, H, D_V, dtype=torch.float32, device=cache.device) if out is None else out
    _need(out, "out", torch.float32, (B, H, D_V), host=True)
    if o_lat is not None:
        _need(o_lat, "o_lat", torch.float32, (B, H, D_C))
    ws = workspace(_lib.OP_DECODE_ATTN, B, L, g=g, w=w, device=cache.device) if ws is None else ws
    rc = _lib.lib().lca_decode_stored_varlen(_ptr(cache), _ptr(rep), rep.shape[1], _ptr(lens), _ptr(q),
                                             _ptr(w_uv), B, L, _params(g, w, scale, 0, pitch), _ptr(out),
                                             _ptr(o_lat), _ptr(ws), ws.numel(), _stream(stream))
    check(rc, "lca_decode_stored_varlen")
    return out


def shard_record_floats(B: int) -> int:
    """Floats in one shard record: o [B][16][512] then lse2 [B][16]."""
    return B * H * _lib.SHARD_RECORD_PER_HEAD


def lca_decode_shard(cache_shard, q_recent, q, L, row0, g=16, w=1024, scale=None, part=None,
                     anchor=None, ws=None, stream=None):
    """Partial decode attention over rows row0 .. row0 + L_shard - 1 of a
    cache of length L (cache_shard [B, L_shard, 576]); returns the shard
    record (float32 [B*16*513]: o, then lse2)."""
    B, Ls, _ = cache_shard.shape
    pitch = _cache(cache_shard, "cache_shard")
    _need(q, "q", torch.bfloat16, (B, H, D))
    if q_recent is not None:
        _need(q_recent, "q_recent", torch.bfloat16, (B, g, H, D))
    dev = cache_shard.device
    part = torch.empty(shard_record_floats(B), dtype=torch.float32, device=dev) if part is None else part
    _need(part, "part", torch.float32, (shard_record_floats(B),))
    if anchor is not None:
        _need(anchor, "anchor", torch.int32)
    ws = workspace(_lib.OP_DECODE, B, L, g=g, w=w, device=dev) if ws is None else ws
    rc = _lib.lib().lca_decode_shard(_ptr(cache_shard), _ptr(q_recent), _ptr(q), B, L, row0, Ls,
                                     _params(g, w, scale, 0, pitch), _ptr(part), _ptr(anchor), _ptr(ws),
                                     ws.numel(), _stream(stream))
    check(rc, "lca_decode_shard")
    return part


def lca_combine_shards(parts, w_uv, B, out=None, o_lat=None, stream=None):
    """parts [n, B*16*513] float32 shard records -> out [B, 16, 128]."""
    n = parts.shape[0]
    _need(parts, "parts", torch.float32, (n, shard_record_floats(B)))
    _need(w_uv, "w_uv", torch.bfloat16, (H, D_C, D_V))
    out = torch.empty(B, H, D_V, dtype=torch.float32, device=parts.device) if out is None else out
    _need(out, "out", torch.float32, (B, H, D_V), host=True)
    if o_lat is not None:
        _need(o_lat, "o_lat", torch.float32, (B, H, D_C))
    rc = _lib.lib().lca_combine_shards(_ptr(parts), n, B, _ptr(w_uv), _ptr(out), _ptr(o_lat),
                                       _stream(stream))
    check(rc, "lca_combine_shards")
    return out


def lca_prefill_block(cache, q, w_uv, q_start, q_len, g=16, w=1024, scale=None, out=None,
                      o_lat=None, anchor=None, ws=None, stream=None, variant=0):
    B, L, _ = cache.shape
    pitch = _cache(cache)
    _need(q, "q", torch.bfloat16, (B, L, H, D))
    _need(w_uv, "w_uv", torch.bfloat16, (H, D_C, D_V))
    out = (torch.empty(B, q_len, H, D_V, dtype=torch.float32, device=cache.device)
           if out is None else out)
    _need(out, "out", torch.float32, (B, q_len, H, D_V), host=True)
    if o_lat is not None:
        _need(o_lat, "o_lat", torch.float32, (B, q_len, H, D_C))
    if anchor is not None:
        _need(anchor, "anchor", torch.int32)
    ws = workspace(_lib.OP_PREFILL, B, L, q_len, g=g, w=w, device=cache.device) if ws is None else ws
    rc = _lib.lib().lca_prefill_block(_ptr(cache), _ptr(q), _ptr(w_uv), B, L, q_start, q_len,
                                      _params(g, w, scale, variant, pitch), _ptr(out), _ptr(o_lat), _ptr(anchor),
                                      _ptr(ws), ws.numel(), _stream(stream))
    check(rc, "lca_prefill_block")
    return out


def lca_append_token(cache, pos, rows, q=None, ring=None, slot=0, q_out=None, stream=None):
    """A decode loop's per-step bookkeeping in one launch: rows [B, 576] go
    into row `pos` of each sequence of `cache` ([B, L, 576], packed or a view
    of a larger [B, L_max, 576] buffer whose rows are contiguous), and, if
    given, the queries q [B, 16, 576] into slot `slot` of `ring`
    [B, g, 16, 576] (the q_recent of the next decode call) and into q_out
    [B, 16, 576] (the q of the next decode call).  rows and q may be pinned
    host tensors: the kernel reads them in place, in lieu of a copy."""
    if not isinstance(cache, torch.Tensor) or not cache.is_cuda or cache.dtype != torch.bfloat16:
        raise TypeError("cache must be a CUDA bfloat16 tensor")
    if cache.dim() != 3 or cache.shape[2] != D or cache.stride(2) != 1 or cache.stride(1) != D:
        raise ValueError(f"cache must be [B, L, {D}] with contiguous rows")
    B, L, _ = cache.shape
    if cache.stride(0) % D or cache.stride(0) < L * D:
        raise ValueError(f"cache must hold each sequence's rows contiguously (strides {cache.stride()})")
    pitch = cache.stride(0) // D
    if not 0 <= pos < L:
        raise ValueError(f"pos {pos} outside the cache's {L} rows")
    _need(rows, "rows", torch.bfloat16, (B, D), host=True)
    g = 0
    if q is not None or ring is not None or q_out is not None:
        _need(q, "q", torch.bfloat16, (B, H, D), host=True)
        if not isinstance(ring, torch.Tensor) or ring.dim() != 4:
            raise ValueError("ring must be [B, g, 16, 576]")
        g = ring.shape[1]
        _need(ring, "ring", torch.bfloat16, (B, g, H, D))
        if q_out is not None:
            _need(q_out, "q_out", torch.bfloat16, (B, H, D))
    rc = _lib.lib().lca_append_token(_ptr(rows), _ptr(cache), B, pitch, int(pos), _ptr(q), _ptr(ring), g,
                                     int(slot), _ptr(q_out), _stream(stream))
    check(rc, "lca_append_token")


def device_status(clear: bool = True) -> tuple[int, int]:
    d = ctypes.c_int(0)
    rc = _lib.lib().lca_device_status(1 if clear else 0, ctypes.byref(d))
    return rc, d.value


def profile_enable(on: bool = True) -> None:
    check(_lib.lib().lca_profile_enable(1 if on else 0), "lca_profile_enable")


def profile_collect() -> dict:
    arr = (_lib.KernelTime * 16)()
    n = _lib.lib().lca_profile_collect(arr, 16)
    if n < 0:
        check(n, "lca_profile_collect")
    return {arr[i].name.decode(): (arr[i].launches, arr[i].total_ms) for i in range(n)}


def launch_count() -> int:
    return int(_lib.lib().lca_launch_count())
